// bitnet_capi.cu -- the extern "C" boundary of libbitnet_b200.so: argument
// validation, workspace layout, launch planning and kernel launches for the
// BitNet b1.58 BitLinear forward.  The operations and their citations are
// documented in include/bitnet_b200.h; the kernels are in the .cuh files
// included below (one translation unit, so the device status word is a
// single symbol).
#include "bitnet_b200.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "act_quant.cuh"
#include "bitdelta.cuh"
#include "common.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "gemv_tiled.cuh"
#include "group_quant.cuh"
#include "peak.cuh"
#include "tiled.cuh"
#include "warmup.cuh"
#include "weight_quant.cuh"

namespace bitnet {

// First failure recorded by a kernel's bounded wait (per device).
__device__ int g_device_status;

namespace {

constexpr int kMaxDevices = 64;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

cudaStream_t as_stream(bitnet_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// The last CUDA error a call of this thread met (0 = none since the last
// query), for bitnet_last_cuda_error.
thread_local int g_last_cuda_error = 0;

bitnet_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return BITNET_OK;
  g_last_cuda_error = static_cast<int>(e);
  return BITNET_ERR_CUDA;
}

bitnet_status launch_status() { return cuda_status(cudaGetLastError()); }

// ------------------------------------------------------------ per-device state

struct DeviceState {
  std::once_flag once;
  bool ok = false;
  int* status = nullptr;  // device address of g_device_status
  int num_sms = 148;
  int gemv_occ[2] = {1, 1};  // resident decode-GEMV CTAs per SM (1 / 2 token tiles)
};
DeviceState g_dev[kMaxDevices];

// Dynamic shared-memory opt-in, and the largest shared-memory carve-out for
// every kernel: kernels that follow one another on an SM then share one L1 /
// shared split, so an SM need not drain to switch between them (the decode
// matmul starts early, next to the activation-quant kernel it depends on).
template <typename K>
bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
             cudaSuccess &&
         cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                              cudaSharedmemCarveoutMaxShared) == cudaSuccess;
}

// Set up the current device once: status-word address, SM count, and the
// shared-memory opt-in of every kernel instance.
DeviceState* device_state() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceState& st = g_dev[dev];
  std::call_once(st.once, [&st, dev]() {
    bool ok = cudaGetSymbolAddress(reinterpret_cast<void**>(&st.status), g_device_status) ==
              cudaSuccess;
    ok = ok && cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev) ==
                   cudaSuccess;
    ok = ok && set_smem(ternary_gemv_kernel<1>, gemv_smem_bytes(1));
    ok = ok && set_smem(ternary_gemv_kernel<2>, gemv_smem_bytes(2));
    for (int nt = 0; nt < 2 && ok; ++nt) {
      int occ = 0;
      ok = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
               &occ, nt ? ternary_gemv_kernel<2> : ternary_gemv_kernel<1>, kGemvThreads,
               gemv_smem_bytes(nt + 1)) ==
           cudaSuccess;
      st.gemv_occ[nt] = std::max(1, occ);
    }
    ok = ok && set_smem(rmsnorm_quant_kernel<true, true, true>, kQuantStageMax);
    ok = ok && set_smem(rmsnorm_quant_kernel<true, false, true>, kQuantStageMax);
    ok = ok && set_smem(rmsnorm_quant_kernel<false, true, true>, kQuantStageMax);
    ok = ok && set_smem(rmsnorm_quant_kernel<false, false, true>, kQuantStageMax);
    ok = ok && set_smem(rmsnorm_quant_grouped_kernel<true>, kQuantStageMax);
    ok = ok && set_smem(rmsnorm_quant_grouped_kernel<false>, 0);
    ok = ok && set_smem(rmsnorm_quant_kernel<true, true, false>, 0);
    ok = ok && set_smem(rmsnorm_quant_kernel<true, false, false>, 0);
    ok = ok && set_smem(rmsnorm_quant_kernel<false, true, false>, 0);
    ok = ok && set_smem(rmsnorm_quant_kernel<false, false, false>, 0);
    ok = ok && set_smem(interleave_rowsum_kernel, 0);
    ok = ok && set_smem(ternary_gemm_tc_kernel<16, false>, GemmCfg<16>::SMEM_DYN);
    ok = ok && set_smem(ternary_gemm_tc_kernel<32, false>, GemmCfg<32>::SMEM_DYN);
    ok = ok && set_smem(ternary_gemm_tc_kernel<64, false>, GemmCfg<64>::SMEM_DYN);
    ok = ok && set_smem(ternary_gemm_tc_kernel<128, false>, GemmCfg<128>::SMEM_DYN);
    ok = ok && set_smem(ternary_gemm_tc_kernel<256, false>, GemmCfg<256>::SMEM_DYN);
    ok = ok && set_smem(ternary_gemm_tc_kernel<16, true>, GemmCfg<16>::SMEM_DYN);
    ok = ok && set_smem(ternary_gemm_tc_kernel<32, true>, GemmCfg<32>::SMEM_DYN);
    ok = ok && set_smem(ternary_gemm_tc_kernel<64, true>, GemmCfg<64>::SMEM_DYN);
    ok = ok && set_smem(ternary_gemm_tc_kernel<128, true>, GemmCfg<128>::SMEM_DYN);
    ok = ok && set_smem(ternary_gemm_tc_kernel<256, true>, GemmCfg<256>::SMEM_DYN);
    ok = ok && set_smem(mma_i8_peak_kernel<false>, kPeakSmem);
    ok = ok && set_smem(mma_i8_peak_kernel<true>, kPeakSmem);
    ok = ok && set_smem(ternary_gemv_tiled_kernel<1, false>, GtCfg<false, 1>::SMEM_DYN);
    ok = ok && set_smem(ternary_gemv_tiled_kernel<2, false>, GtCfg<false, 2>::SMEM_DYN);
    ok = ok && set_smem(ternary_gemv_tiled_kernel<1, true>, GtCfg<true, 1>::SMEM_DYN);
    ok = ok && set_smem(ternary_gemv_tiled_kernel<2, true>, GtCfg<true, 2>::SMEM_DYN);
    st.ok = ok;
  });
  return st.ok ? &st : nullptr;
}

// --------------------------------------------------------------- TMA maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D uint8 tensor [rows][inner] with the given row stride (bytes), boxes
// of box_rows x box_inner; out-of-range elements read as zero.
bool make_tmap_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                  uint64_t row_stride, uint32_t box_inner, uint32_t box_rows,
                  CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// -------------------------------------------------------- workspace layout

struct FwdWorkspace {
  size_t xq, sx, rs, acc, cnt, total;
};

constexpr int64_t kGemvMaxM = 16;
// Token counts up to this one are "decode-sized" for the tcgen05 kernel too:
// it splits K across CTAs to fill the GPU and needs the partial-sum region.
constexpr int64_t kSplitMaxM = 64;

// Workspace of one forward.  The quantized input takes M * 256 * ceil(K/256)
// bytes: row-major [M][K] for the tcgen05 kernel and the row-major decode
// kernel, chunk-major [K/256][M][256] (zero-padded past K) for the tiled
// decode kernel.  For M <= 16 the partial-sum region serves either decode
// kernel: the row-major one accumulates [M][N] int32 split-K partials with
// atomics, the tiled one stores [M][128] int32 partial slots, two per CTA
// that touches the problem; the counters follow it.
FwdWorkspace fwd_layout(int64_t M, int64_t N, int64_t K) {
  FwdWorkspace w{};
  size_t o = 0;
  w.xq = o;
  o = align256(o + static_cast<size_t>(M * 256 * tiled_chunks(K)));
  w.sx = o;
  o = align256(o + 4 * static_cast<size_t>(M));
  w.rs = o;
  o = align256(o + 4 * static_cast<size_t>(M));
  const bool split_capable = M <= kSplitMaxM;
  const int64_t tiles = tiled_row_blocks(N) * tiled_chunks(K);
  const size_t slots =
      M <= kGemvMaxM ? 2 * static_cast<size_t>(std::min<int64_t>(kGtMaxCtas, tiles)) : 0;
  w.acc = o;
  o = align256(o + (split_capable ? std::max(4 * static_cast<size_t>(M * N),
                                             slots * kTileRows * 4 * static_cast<size_t>(M))
                                  : 0));
  w.cnt = o;
  o = align256(o + (split_capable ? 4 * static_cast<size_t>(std::max<int64_t>((N + 15) / 16,
                                                                               tiled_row_blocks(N)))
                                  : 0));
  w.total = o;
  return w;
}

// ---------------------------------------------------------------- checks

bitnet_status check_shape(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return BITNET_ERR_INVALID_ARG;
  if (N < 1 || N > BITNET_MAX_N || M > BITNET_MAX_M) return BITNET_ERR_UNSUPPORTED_SHAPE;
  if (K < 64 || K > BITNET_MAX_K || (K % 64) != 0) return BITNET_ERR_UNSUPPORTED_SHAPE;
  return BITNET_OK;
}

bool ok_dtype(int d) { return d == BITNET_F32 || d == BITNET_BF16; }

// ------------------------------------------------------------ launchers

// ------------------------------------------------------------ decode GEMV

// Work a stream-K launch loses to its cross-CTA finish (partials through
// the workspace, a fence, a counter, a read-back), in 4 KiB units per CTA.
constexpr long long kGemvSplitPenaltyUnits = 24;

// Relative time of one unit: two token tiles take about 1.2 times as long as
// one (fitted to in-kernel timestamps of the decode shapes).
long long gemv_unit_cost(const GemvProblem& P) { return P.M > 8 ? 6 : 5; }

// Deal whole row blocks, largest first, to the least-loaded CTA (at most
// kGemvMaxSegs each).  Returns the largest CTA load in units, or -1 when
// the launch does not fit the explicit list.
long long plan_gemv_listed(GemvLaunch& L, long long G) {
  int total = 0;
  for (int i = 0; i < L.count; ++i) total += L.prob[i].rb;
  if (total > G * kGemvMaxSegs || G > kGemvMaxCtas || G < 1 || total >= 65536) return -1;
  // Problems by decreasing row-block size.
  int order[kGemvMaxGroup];
  for (int i = 0; i < L.count; ++i) order[i] = i;
  std::sort(order, order + L.count, [&L](int a, int b) {
    return gemv_unit_cost(L.prob[a]) * L.prob[a].kc > gemv_unit_cost(L.prob[b]) * L.prob[b].kc;
  });
  // Min-heap of (load, cta).
  std::vector<std::pair<long long, int>> heap;
  heap.reserve(static_cast<size_t>(G));
  for (int c = 0; c < G; ++c) heap.emplace_back(0LL, c);
  std::vector<std::vector<uint16_t>> lists(static_cast<size_t>(G));
  auto cmp = [](const std::pair<long long, int>& a, const std::pair<long long, int>& b) {
    return a.first != b.first ? a.first > b.first : a.second > b.second;
  };
  std::make_heap(heap.begin(), heap.end(), cmp);
  long long worst = 0;
  for (int oi = 0; oi < L.count; ++oi) {
    const GemvProblem& P = L.prob[order[oi]];
    for (int r = 0; r < P.rb; ++r) {
      if (heap.empty()) return -1;
      std::pop_heap(heap.begin(), heap.end(), cmp);
      auto top = heap.back();
      heap.pop_back();
      lists[static_cast<size_t>(top.second)].push_back(static_cast<uint16_t>(P.rb_begin + r));
      top.first += gemv_unit_cost(P) * P.kc;
      worst = std::max(worst, top.first);
      if (lists[static_cast<size_t>(top.second)].size() < static_cast<size_t>(kGemvMaxSegs)) {
        heap.push_back(top);
        std::push_heap(heap.begin(), heap.end(), cmp);
      }
    }
  }
  for (long long c = 0; c < G; ++c) {
    auto& v = lists[static_cast<size_t>(c)];
    std::sort(v.begin(), v.end());
    L.ntask[c] = static_cast<uint8_t>(v.size());
    for (size_t i = 0; i < v.size(); ++i) L.task[c][i] = v[i];
  }
  return worst;
}

// Shape fields of prob[0..count) must be set.  Lays the problems' units end
// to end and returns the CTA count.  Whole row blocks per CTA when that
// balances within the cost of splitting; otherwise stream-K: one CTA per 8
// units (a unit per warp) up to the resident capacity, and enough CTAs that
// no CTA's share touches more than kGemvMaxSegs row blocks.
long long plan_gemv_launch(GemvLaunch& L, long long capacity) {
  long long U = 0;
  int rbs = 0, kc_min = 1 << 30;
  for (int i = 0; i < L.count; ++i) {
    GemvProblem& P = L.prob[i];
    P.rb = (P.N + kGemvRows - 1) / kGemvRows;
    P.kc = (P.K + kGemvUnitK - 1) / kGemvUnitK;
    P.unit_begin = U;
    P.rb_begin = rbs;
    U += static_cast<long long>(P.rb) * P.kc;
    rbs += P.rb;
    kc_min = std::min(kc_min, P.kc);
  }
  L.units = U;
  capacity = std::max(1LL, capacity);
  long long G = std::min((U + kGemvWarps - 1) / kGemvWarps, capacity);
  // A share of n <= (kGemvMaxSegs - 1) * kc_min units touches at most
  // kGemvMaxSegs row blocks.
  const long long per = static_cast<long long>(kGemvMaxSegs - 1) * kc_min;
  G = std::max(G, (U + per - 1) / per);
  G = std::max(1LL, std::min(G, U));
  long long W = 0;  // total weighted cost
  for (int i = 0; i < L.count; ++i)
    W += gemv_unit_cost(L.prob[i]) * static_cast<long long>(L.prob[i].rb) * L.prob[i].kc;
  // CTAs beyond the resident capacity run as a later wave: cost per wave.
  const long long waves = (G + capacity - 1) / capacity;
  const long long split_cost = waves * ((W + G - 1) / G + 2 * kGemvSplitPenaltyUnits);
  const long long Gl = std::min<long long>(capacity, rbs);
  const long long listed_cost = plan_gemv_listed(L, Gl);
  if (listed_cost >= 0 && listed_cost <= split_cost) {
    L.listed = 1;
    return Gl;
  }
  L.listed = 0;
  return G;
}

// Whether a CTA boundary of a G-CTA launch falls inside a row block of
// problem i (its partials then go through the workspace, which must start
// at zero).
bool gemv_problem_shared(const GemvLaunch& L, int i, long long G) {
  if (L.listed) return false;
  const GemvProblem& P = L.prob[i];
  const long long U = L.units, lo = P.unit_begin, hi = lo + static_cast<long long>(P.rb) * P.kc;
  for (long long b = gemv_cta_of(lo, U, G) + 1; b <= gemv_cta_of(hi - 1, U, G); ++b)
    if ((b * U / G - lo) % P.kc != 0) return true;
  return false;
}

// The activation box has the problem's own token tiles (8 or 16 rows).
// xws / xL: the workspace holding this problem's quantized activations (its
// own, or that of an earlier problem of the launch with the same input);
// ws / L: its own workspace (split-K partials).
bool fill_gemv_problem(GemvMaps& maps, GemvProblem& q, const uint8_t* Wp, uint8_t* xws,
                       const FwdWorkspace& xL, uint8_t* ws, const FwdWorkspace& L,
                       const float* s_x, const float* s_w, int64_t M, int64_t N, int64_t K,
                       void* y, int y_dtype, int32_t* acc_out) {
  // One unit = a 64-row x 64-byte weight box and a 256-byte x 8 nt-row
  // activation box; rows past N or M and bytes past K read as zero.
  if (!make_tmap_u8(&maps.tmap_w, Wp, static_cast<uint64_t>(K / 4), static_cast<uint64_t>(N),
                    static_cast<uint64_t>(K / 4), kGemvUnitK / 4, kGemvRows,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
    return false;
  if (!make_tmap_u8(&maps.tmap_x, xws + xL.xq, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                    static_cast<uint64_t>(K), kGemvUnitK, M > 8 ? 16u : 8u,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
    return false;
  q.W = Wp;
  q.xq = reinterpret_cast<const int8_t*>(xws + xL.xq);
  q.rowsum = reinterpret_cast<const int32_t*>(xws + xL.rs);
  q.s_x = s_x;
  q.s_w = s_w;
  q.y = y;
  q.acc_out = acc_out;
  q.ws_acc = reinterpret_cast<int32_t*>(ws + L.acc);
  q.ws_cnt = reinterpret_cast<unsigned*>(ws + L.cnt);
  q.M = static_cast<int>(M);
  q.N = static_cast<int>(N);
  q.K = static_cast<int>(K);
  q.y_bf16 = (y_dtype == BITNET_BF16) ? 1 : 0;
  return true;
}

// Token tiles of a launch: two n8 tiles when any problem has more than 8.
int gemv_tiles(const GemvLaunch& L) {
  for (int i = 0; i < L.count; ++i)
    if (L.prob[i].M > 8) return 2;
  return 1;
}

bitnet_status launch_gemv_group(const DeviceState& ds, GemvLaunch& L, long long G, bool pdl,
                                bool early_weights, cudaStream_t stream) {
  L.use_pdl = pdl ? 1 : 0;
  L.early_weights = (pdl && early_weights) ? 1 : 0;
  L.status = ds.status;
  L.wait_limit_ns = kWaitLimitNs;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(G), 1, 1);
  cfg.blockDim = dim3(kGemvThreads, 1, 1);
  const int nt = gemv_tiles(L);
  cfg.dynamicSmemBytes = gemv_smem_bytes(nt);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const cudaError_t e = nt == 2 ? cudaLaunchKernelEx(&cfg, ternary_gemv_kernel<2>, L)
                                : cudaLaunchKernelEx(&cfg, ternary_gemv_kernel<1>, L);
  return cuda_status(e);
}

long long gemv_capacity(const DeviceState& ds, int M) {
  return static_cast<long long>(ds.num_sms) * (M > 8 ? ds.gemv_occ[1] : ds.gemv_occ[0]);
}

// One problem: its plan (count = 1) in *L.
long long plan_gemv_single(const DeviceState& ds, GemvLaunch& L, int64_t M, int64_t N,
                           int64_t K) {
  L.count = 1;
  L.prob[0].M = static_cast<int>(M);
  L.prob[0].N = static_cast<int>(N);
  L.prob[0].K = static_cast<int>(K);
  return plan_gemv_launch(L, gemv_capacity(ds, static_cast<int>(M)));
}

bitnet_status launch_gemv(const DeviceState& ds, const uint8_t* Wp, const float* s_x,
                          const float* s_w, int64_t M, int64_t N, int64_t K, uint8_t* ws,
                          const FwdWorkspace& Lw, void* y, int y_dtype, int32_t* acc_out,
                          bool pdl, bool early_weights, cudaStream_t stream) {
  static thread_local GemvLaunch L;  // ~9 KB: keep it off the stack
  if (!fill_gemv_problem(L.maps[0], L.prob[0], Wp, ws, Lw, ws, Lw, s_x, s_w, M, N, K, y, y_dtype,
                         acc_out))
    return BITNET_ERR_CUDA;
  const long long G = plan_gemv_single(ds, L, M, N, K);
  return launch_gemv_group(ds, L, G, pdl, early_weights, stream);
}

// ------------------------------------------------------ tiled decode GEMV

// Relative time of one 8 KiB tile: two token tiles take about 1.2 times as
// long as one (the same weights as the row-major kernel's cost model).
long long gt_tile_cost(const GtProblem& P) { return P.M > 8 ? 6 : 5; }

// Shape fields (M, N, K) of prob[0..count) must be set.  Lays the problems'
// tiles end to end and splits them into `capacity` (at most the tile count)
// contiguous ranges of equal cost; every range holds at least one tile.
void plan_gt_launch(GtLaunch& L, long long capacity) {
  long long T = 0, W = 0;
  for (int i = 0; i < L.count; ++i) {
    GtProblem& P = L.prob[i];
    P.KC = static_cast<int>(tiled_chunks(P.K));
    P.RB = static_cast<int>(tiled_row_blocks(P.N));
    P.tile_base = T;
    const long long tiles = static_cast<long long>(P.RB) * P.KC;
    T += tiles;
    W += tiles * gt_tile_cost(P);
  }
  long long G = std::max(1LL, std::min({capacity, T, static_cast<long long>(kGtMaxCtas)}));
  L.ctas = static_cast<int>(G);
  // tile_begin[b]: first tile whose cost prefix reaches b * W / G.
  int p = 0;
  long long pre = 0;  // cost of the tiles before problem p
  for (long long b = 0; b <= G; ++b) {
    const long long target = (b * W + G - 1) / G;
    while (p + 1 < L.count &&
           pre + (static_cast<long long>(L.prob[p].RB) * L.prob[p].KC) * gt_tile_cost(L.prob[p]) <
               target) {
      pre += static_cast<long long>(L.prob[p].RB) * L.prob[p].KC * gt_tile_cost(L.prob[p]);
      ++p;
    }
    const long long c = gt_tile_cost(L.prob[p]);
    long long t = L.prob[p].tile_base + (target - pre + c - 1) / c;
    L.tile_begin[b] = std::min(t, T);
  }
  L.tile_begin[0] = 0;
  L.tile_begin[G] = T;
  for (long long b = 1; b < G; ++b)  // strictly increasing, room for the rest
    L.tile_begin[b] = std::min(std::max(L.tile_begin[b], L.tile_begin[b - 1] + 1), T - (G - b));
  for (int i = 0; i < L.count; ++i) {
    GtProblem& P = L.prob[i];
    int b = 0;
    while (b + 1 < G && L.tile_begin[b + 1] <= P.tile_base) ++b;
    P.cta_first = b;
  }
}

bool fill_gt_problem(GtProblem& q, const uint8_t* Wt, uint8_t* xws, const FwdWorkspace& xL,
                     uint8_t* ws, const FwdWorkspace& Lw, const float* s_x, const float* s_w,
                     int64_t M, int64_t N, int64_t K, void* y, int y_dtype, int32_t* acc_out) {
  q.Wt = Wt;
  q.xd = xws + xL.xq;
  q.rowsum = reinterpret_cast<const int32_t*>(xws + xL.rs);
  q.s_x = s_x;
  q.s_w = s_w;
  q.y = y;
  q.acc_out = acc_out;
  q.part = reinterpret_cast<int32_t*>(ws + Lw.acc);
  q.M = static_cast<int>(M);
  q.N = static_cast<int>(N);
  q.K = static_cast<int>(K);
  q.y_bf16 = (y_dtype == BITNET_BF16) ? 1 : 0;
  q.s_w2 = nullptr;
  q.gc = 0;
  q.G = 1;
  q.gacc = nullptr;
  return true;
}

int gt_tiles(const GtLaunch& L) {
  for (int i = 0; i < L.count; ++i)
    if (L.prob[i].M > 8) return 2;
  return 1;
}

// Whether a row block (with group-wise scales: a row-block group) of L is
// split between CTAs: then the fixup kernel has to add the parts.  A CTA
// range that starts where no such span starts splits one.
bool gt_needs_fixup(const GtLaunch& L) {
  int p = 0;
  for (int b = 1; b < L.ctas; ++b) {
    const long long t = L.tile_begin[b];
    while (p + 1 < L.count && t >= L.prob[p + 1].tile_base) ++p;
    const GtProblem& P = L.prob[p];
    const long long c = (t - P.tile_base) % P.KC;
    if (c % (P.gc > 0 ? P.gc : P.KC) != 0) return true;
  }
  return false;
}

// pair: the fused SwiGLU variant (every problem of L has pair-tiled weights).
// The streaming kernel, then (when a span is split) the fixup kernel as its
// programmatic dependent.
bitnet_status launch_gt(const DeviceState& ds, GtLaunch& L, bool pdl, cudaStream_t stream,
                        bool pair = false) {
  L.use_pdl = pdl ? 1 : 0;
  L.status = ds.status;
  L.wait_limit_ns = kWaitLimitNs;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(L.ctas), 1, 1);
  cfg.blockDim = dim3(kGtThreads, 1, 1);
  const int nt = gt_tiles(L);
  cfg.dynamicSmemBytes = pair ? (nt == 2 ? GtCfg<true, 2>::SMEM_DYN : GtCfg<true, 1>::SMEM_DYN)
                              : (nt == 2 ? GtCfg<false, 2>::SMEM_DYN : GtCfg<false, 1>::SMEM_DYN);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e;
  if (pair)
    e = nt == 2 ? cudaLaunchKernelEx(&cfg, ternary_gemv_tiled_kernel<2, true>, L)
                : cudaLaunchKernelEx(&cfg, ternary_gemv_tiled_kernel<1, true>, L);
  else
    e = nt == 2 ? cudaLaunchKernelEx(&cfg, ternary_gemv_tiled_kernel<2, false>, L)
                : cudaLaunchKernelEx(&cfg, ternary_gemv_tiled_kernel<1, false>, L);
  if (e != cudaSuccess || !gt_needs_fixup(L)) return cuda_status(e);
  int mmax = 1;
  for (int i = 0; i < L.count; ++i) mmax = std::max(mmax, L.prob[i].M);
  cfg.gridDim = dim3(static_cast<unsigned>(L.ctas),
                     static_cast<unsigned>((mmax + kGtFixTokens - 1) / kGtFixTokens), 1);
  cfg.blockDim = dim3(kTileRows * kGtFixTokens, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.numAttrs = 1;
  e = pair ? cudaLaunchKernelEx(&cfg, gemv_tiled_fixup_kernel<true>, L)
           : cudaLaunchKernelEx(&cfg, gemv_tiled_fixup_kernel<false>, L);
  return cuda_status(e);
}

// One problem on tiled weights.
bitnet_status launch_gt_single(const DeviceState& ds, const uint8_t* Wt, const float* s_x,
                               const float* s_w, int64_t M, int64_t N, int64_t K, uint8_t* ws,
                               const FwdWorkspace& Lw, void* y, int y_dtype, int32_t* acc_out,
                               bool pdl, cudaStream_t stream) {
  static thread_local GtLaunch L;  // ~6 KB: keep it off the stack
  L.count = 1;
  fill_gt_problem(L.prob[0], Wt, ws, Lw, ws, Lw, s_x, s_w, M, N, K, y, y_dtype, acc_out);
  plan_gt_launch(L, ds.num_sms);
  return launch_gt(ds, L, pdl, stream);
}

struct GemmPlan {
  int BN, rb, tb, ksplit, steps_per_split;
};

// Token tile BN from M (and K: above 128 tokens, 128-token tiles two per
// SM while K <= 8192 or M <= 1024, where per-tile pipeline fill and
// epilogue dominate; 256-token tiles otherwise -- measured on the prefill
// shapes).  K is
// split across CTAs only for small M (then the int32 partials go through the
// workspace), to give every SM work.
GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int num_sms) {
  GemmPlan pl{};
  pl.BN = M <= 16 ? 16
        : (M <= 32 ? 32 : (M <= 64 ? 64 : (M <= 1024 || K <= 8192 ? 128 : 256)));
  pl.rb = static_cast<int>((N + 127) / 128);
  pl.tb = static_cast<int>((M + pl.BN - 1) / pl.BN);
  const bool small = pl.BN <= 128;           // GemmCfg<BN>::TWO_PER_SM
  const int kstep = 256;                      // GemmCfg<BN>::KSTEP
  const int steps = static_cast<int>((K + kstep - 1) / kstep);
  int ks = 1;
  if (M <= kSplitMaxM) {
    // Resident slots: two CTAs per SM for small token tiles.  Split K so the
    // grid fills the slots without starting a partial second wave.
    const int slots = (small ? 2 : 1) * num_sms;
    const int tiles = pl.rb * pl.tb;
    if (tiles < slots) ks = std::max(1, std::min(steps, slots / tiles));
  }
  pl.steps_per_split = (steps + ks - 1) / ks;
  pl.ksplit = (steps + pl.steps_per_split - 1) / pl.steps_per_split;
  return pl;
}

template <int BN>
bitnet_status launch_gemm_bn(const CUtensorMap& tx, const CUtensorMap& tw, const GemmParams& p,
                             const GemmPlan& pl, bool tiled_w, cudaStream_t stream) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.rb), static_cast<unsigned>(pl.tb),
                     static_cast<unsigned>(pl.ksplit));
  cfg.blockDim = dim3(GemmCfg<BN>::THREADS, 1, 1);
  cfg.dynamicSmemBytes = GemmCfg<BN>::SMEM_DYN;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.use_pdl ? 1 : 0;
  const cudaError_t e = tiled_w ? cudaLaunchKernelEx(&cfg, ternary_gemm_tc_kernel<BN, true>, tx, tw, p)
                                : cudaLaunchKernelEx(&cfg, ternary_gemm_tc_kernel<BN, false>, tx, tw, p);
  return cuda_status(e);
}

// Wp: row-major packed weights, or the tiled layout when tiled_w.
bitnet_status launch_gemm(const DeviceState& ds, const uint8_t* Wp, const int8_t* xi,
                          const int32_t* rowsum, const float* s_x, const float* s_w, int64_t M,
                          int64_t N, int64_t K, uint8_t* ws, const FwdWorkspace& Lw, void* y,
                          int y_dtype, int32_t* acc_out, bool pdl, cudaStream_t stream,
                          bool tiled_w = false) {
  const GemmPlan pl = plan_gemm(M, N, K, ds.num_sms);
  CUtensorMap tx, tw;
  if (!make_tmap_u8(&tx, xi, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                    static_cast<uint64_t>(K), 128, static_cast<uint32_t>(pl.BN),
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return BITNET_ERR_CUDA;
  // GemmCfg<BN>::WP_ROW = 64 bytes per row, swizzled so the unpack reads are
  // bank-conflict free (the tiled layout is stored in that order already).
  if (tiled_w)
    std::memset(&tw, 0, sizeof(tw));
  else if (!make_tmap_u8(&tw, Wp, static_cast<uint64_t>(K / 4), static_cast<uint64_t>(N),
                         static_cast<uint64_t>(K / 4), 64, 128, CU_TENSOR_MAP_SWIZZLE_64B))
    return BITNET_ERR_CUDA;
  GemmParams p{};
  p.Wt = tiled_w ? Wp : nullptr;
  p.KC = static_cast<int>(tiled_chunks(K));
  p.rowsum = rowsum;
  p.s_x = s_x;
  p.s_w = s_w;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.y = y;
  p.y_bf16 = (y_dtype == BITNET_BF16) ? 1 : 0;
  p.acc_out = acc_out;
  p.ksplit = pl.ksplit;
  p.steps_per_split = pl.steps_per_split;
  p.ws_acc = reinterpret_cast<int32_t*>(ws + Lw.acc);
  p.ws_cnt = reinterpret_cast<unsigned*>(ws + Lw.cnt);
  p.status = ds.status;
  p.wait_limit_ns = kWaitLimitNs;
  p.use_pdl = pdl ? 1 : 0;
  switch (pl.BN) {
    case 16: return launch_gemm_bn<16>(tx, tw, p, pl, tiled_w, stream);
    case 32: return launch_gemm_bn<32>(tx, tw, p, pl, tiled_w, stream);
    case 64: return launch_gemm_bn<64>(tx, tw, p, pl, tiled_w, stream);
    case 128: return launch_gemm_bn<128>(tx, tw, p, pl, tiled_w, stream);
    default: return launch_gemm_bn<256>(tx, tw, p, pl, tiled_w, stream);
  }
}

// The tcgen05 kernel in group mode: K split z = group z, each CTA writes its
// group's integer sums (row sums of the group subtracted) to gacc [G][M][N].
bitnet_status launch_gemm_groups(const DeviceState& ds, const uint8_t* Wp, const int8_t* xi,
                                 const int32_t* rowsum, int64_t M, int64_t N, int64_t K,
                                 int64_t G, int32_t* gacc, const GemmPlan& pl, bool tiled_w,
                                 cudaStream_t stream) {
  CUtensorMap tx, tw;
  if (!make_tmap_u8(&tx, xi, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                    static_cast<uint64_t>(K), 128, static_cast<uint32_t>(pl.BN),
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return BITNET_ERR_CUDA;
  if (tiled_w)
    std::memset(&tw, 0, sizeof(tw));
  else if (!make_tmap_u8(&tw, Wp, static_cast<uint64_t>(K / 4), static_cast<uint64_t>(N),
                         static_cast<uint64_t>(K / 4), 64, 128, CU_TENSOR_MAP_SWIZZLE_64B))
    return BITNET_ERR_CUDA;
  GemmParams p{};
  p.Wt = tiled_w ? Wp : nullptr;
  p.KC = static_cast<int>(tiled_chunks(K));
  p.rowsum = rowsum;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.ksplit = pl.ksplit;
  p.steps_per_split = pl.steps_per_split;
  p.status = ds.status;
  p.wait_limit_ns = kWaitLimitNs;
  p.use_pdl = 1;
  p.gacc = gacc;
  p.G = static_cast<int>(G);
  switch (pl.BN) {
    case 16: return launch_gemm_bn<16>(tx, tw, p, pl, tiled_w, stream);
    case 32: return launch_gemm_bn<32>(tx, tw, p, pl, tiled_w, stream);
    case 64: return launch_gemm_bn<64>(tx, tw, p, pl, tiled_w, stream);
    case 128: return launch_gemm_bn<128>(tx, tw, p, pl, tiled_w, stream);
    default: return launch_gemm_bn<256>(tx, tw, p, pl, tiled_w, stream);
  }
}

// Whether the matmul chosen for (path, M, N, K) accumulates split-K partials
// in the workspace (which must then start at zero).
bool needs_zeroed_partials(const DeviceState& ds, int path, int64_t M, int64_t N, int64_t K) {
  if (M > kSplitMaxM) return false;
  if (path == BITNET_PATH_GEMV) {
    static thread_local GemvLaunch L;
    const long long G = plan_gemv_single(ds, L, M, N, K);
    return gemv_problem_shared(L, 0, G);
  }
  return plan_gemm(M, N, K, ds.num_sms).ksplit > 1;
}

// Extra blocks appended to a row-per-block kernel to clear `bytes` bytes.
int64_t zero_blocks(size_t bytes) {
  if (bytes == 0) return 0;
  const int64_t per_block = 16 * kActThreads * 4;  // four 16-byte stores per thread
  return std::min<int64_t>(256, (static_cast<int64_t>(bytes) + per_block - 1) / per_block);
}

// Layouts of the quantized activations a launch writes.
// kXDecode: interleaved + x_block_pos (row-major decode kernel);
// kXDecodeTiled: the same, chunk-major [K/256][M][256] (tiled decode kernel).
enum XLayout { kXNatural = 0, kXInterleaved = 1, kXDecode = 2, kXDecodeTiled = 3 };

// zero/zero_bytes: a 16-byte aligned range (multiple of 16 bytes) cleared by
// extra blocks of the same launch, or null/0.
bitnet_status launch_act_quant(const void* x, int x_dtype, const float* gamma, float eps,
                               int64_t M, int64_t K, int8_t* x_q, float* s_x, int32_t* rowsum,
                               int layout, bool trigger, void* zero, size_t zero_bytes,
                               cudaStream_t stream) {
  const bool interleave = layout != kXNatural;
  const int perm = (layout == kXDecode || layout == kXDecodeTiled) ? 1 : 0;
  const int tiled = layout == kXDecodeTiled ? 1 : 0;
  const int64_t zb = zero ? zero_blocks(zero_bytes) : 0;
  dim3 grid(static_cast<unsigned>(M + zb)), block(kActThreads);
  const int trig = trigger ? 1 : 0;
  uint4* z = static_cast<uint4*>(zero);
  const int64_t n16 = zero ? static_cast<int64_t>(zero_bytes / 16) : 0;
  const bool bf16 = x_dtype == BITNET_BF16;
  const uint32_t stage = quant_stage_bytes(K, bf16, gamma != nullptr);
  const bool staged = stage <= kQuantStageMax;
  int* status = device_state() ? device_state()->status : nullptr;
  const size_t dyn = staged ? stage : 0;
#define BITNET_QUANT(BF, IL, ST)                                                             \
  rmsnorm_quant_kernel<BF, IL, ST><<<grid, block, dyn, stream>>>(                           \
      x, gamma, eps, M, K, x_q, s_x, rowsum, z, n16, trig, status, kWaitLimitNs, perm, tiled)
  if (bf16) {
    if (interleave) {
      if (staged) BITNET_QUANT(true, true, true); else BITNET_QUANT(true, true, false);
    } else {
      if (staged) BITNET_QUANT(true, false, true); else BITNET_QUANT(true, false, false);
    }
  } else {
    if (interleave) {
      if (staged) BITNET_QUANT(false, true, true); else BITNET_QUANT(false, true, false);
    } else {
      if (staged) BITNET_QUANT(false, false, true); else BITNET_QUANT(false, false, false);
    }
  }
#undef BITNET_QUANT
  return launch_status();
}

// The split-K partials + counters of a layout (zero bytes when the layout
// has no partial-sum region).
void* splitk_region(uint8_t* ws, const FwdWorkspace& L, size_t* bytes) {
  *bytes = L.total - L.acc;
  return *bytes ? ws + L.acc : nullptr;
}

// Only the arrival counters: the tiled decode kernel's partial slots are
// written before they are read.
void* counter_region(uint8_t* ws, const FwdWorkspace& L, size_t* bytes) {
  *bytes = L.total - L.cnt;
  return *bytes ? ws + L.cnt : nullptr;
}

// Matmul + fused dequant on already-prepared interleaved activations.
// w_layout: BITNET_LAYOUT_ROWS or BITNET_LAYOUT_TILED (then the decode path
// is the tiled decode kernel, whose activations are chunk-major).
bitnet_status run_matmul(const DeviceState& ds, int path, const uint8_t* Wp, uint8_t* ws,
                         const FwdWorkspace& L, const float* s_x, const float* s_w, int64_t M,
                         int64_t N, int64_t K, void* y, int y_dtype, int32_t* acc_out, bool pdl,
                         bool early_weights, cudaStream_t stream, int w_layout = 0) {
  const bool tiled = w_layout == BITNET_LAYOUT_TILED;
  if (path == BITNET_PATH_GEMV) {
    if (tiled)
      return launch_gt_single(ds, Wp, s_x, s_w, M, N, K, ws, L, y, y_dtype, acc_out, pdl,
                              stream);
    return launch_gemv(ds, Wp, s_x, s_w, M, N, K, ws, L, y, y_dtype, acc_out, pdl,
                       early_weights, stream);
  }
  const int8_t* xi = reinterpret_cast<const int8_t*>(ws + L.xq);
  const int32_t* rs = reinterpret_cast<const int32_t*>(ws + L.rs);
  return launch_gemm(ds, Wp, xi, rs, s_x, s_w, M, N, K, ws, L, y, y_dtype, acc_out, pdl,
                     stream, tiled);
}

// The activation layout the chosen matmul reads.
int x_layout_for(int path, int w_layout) {
  if (path != BITNET_PATH_GEMV) return kXInterleaved;
  return w_layout == BITNET_LAYOUT_TILED ? kXDecodeTiled : kXDecode;
}

// Which part of the workspace the quant launch clears for the chosen matmul.
void* zero_region_for(const DeviceState& ds, int path, int w_layout, int64_t M, int64_t N,
                      int64_t K, uint8_t* ws, const FwdWorkspace& L, size_t* bytes) {
  *bytes = 0;
  if (path == BITNET_PATH_GEMV && w_layout == BITNET_LAYOUT_TILED)
    return counter_region(ws, L, bytes);
  return needs_zeroed_partials(ds, path, M, N, K) ? splitk_region(ws, L, bytes) : nullptr;
}

// Decode GEMV (warp-level MMA) for M <= 16 unless the matrix is large: above
// ~32 MB of packed weights the tcgen05 kernel streams faster (measured on
// B200), and for M > 16 it is the only path.
constexpr int64_t kGemvAutoMaxBytes = int64_t(32) << 20;

// With tiled weights the decode kernel streams any size at full rate, so
// it serves every M <= 16.
int resolve_path(int path, int64_t M, int64_t N = 0, int64_t K = 0, int w_layout = 0) {
  if (path != BITNET_PATH_AUTO) return path;
  if (M > kGemvMaxM) return BITNET_PATH_GEMM;
  if (w_layout == BITNET_LAYOUT_TILED) return BITNET_PATH_GEMV;
  return (N * (K / 4) <= kGemvAutoMaxBytes) ? BITNET_PATH_GEMV : BITNET_PATH_GEMM;
}

bitnet_status forward_impl(const void* x, int x_dtype, const float* gamma, float eps,
                           const uint8_t* W_packed, const float* s_w, int64_t M, int64_t N,
                           int64_t K, void* y, int y_dtype, void* workspace,
                           size_t workspace_bytes, int8_t* x_q_out, float* s_x_out,
                           int32_t* acc_out, int path, cudaStream_t stream, int w_layout = 0) {
  bitnet_status st = check_shape(M, N, K);
  if (st != BITNET_OK) return st;
  if (M == 0) return BITNET_OK;  // empty batch: nothing to read or write
  if (!x || !W_packed || !s_w || !ok_dtype(x_dtype) || !(eps >= 0.0f) || eps > 3.0e38f)
    return BITNET_ERR_INVALID_ARG;
  if (y && !ok_dtype(y_dtype)) return BITNET_ERR_INVALID_ARG;
  if (path < BITNET_PATH_AUTO || path > BITNET_PATH_GEMM) return BITNET_ERR_INVALID_ARG;
  if (w_layout != BITNET_LAYOUT_ROWS && w_layout != BITNET_LAYOUT_TILED)
    return BITNET_ERR_INVALID_ARG;
  path = resolve_path(path, M, N, K, w_layout);
  if (path == BITNET_PATH_GEMV && M > kGemvMaxM) return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || (gamma && !aligned(gamma, 16)) || !aligned(W_packed, 16) ||
      !aligned(s_w, 4) || (y && !aligned(y, 16)) || (x_q_out && !aligned(x_q_out, 16)) ||
      (s_x_out && !aligned(s_x_out, 4)) || (acc_out && !aligned(acc_out, 16)))
    return BITNET_ERR_MISALIGNED;
  const FwdWorkspace L = fwd_layout(M, N, K);
  if (!workspace || workspace_bytes < L.total) return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  if (x_q_out || s_x_out) {
    // Debug export in natural k order (same arithmetic as the fused pass).
    int8_t* xq_nat = x_q_out ? x_q_out : reinterpret_cast<int8_t*>(ws + L.xq);
    st = launch_act_quant(x, x_dtype, gamma, eps, M, K, xq_nat, s_x_out, nullptr, kXNatural,
                          false, nullptr, 0, stream);
    if (st != BITNET_OK) return st;
  }
  const bool pdl = true;  // the matmul launch follows the quant launch directly
  float* sx = reinterpret_cast<float*>(ws + L.sx);
  size_t zbytes = 0;
  void* zero = zero_region_for(*ds, path, w_layout, M, N, K, ws, L, &zbytes);
  st = launch_act_quant(x, x_dtype, gamma, eps, M, K, reinterpret_cast<int8_t*>(ws + L.xq), sx,
                        reinterpret_cast<int32_t*>(ws + L.rs), x_layout_for(path, w_layout), pdl,
                        zero, zbytes, stream);
  if (st != BITNET_OK) return st;
  // The activation-quant kernel just queued started after every earlier
  // write to W_packed, so the GEMV may fetch weights before waiting on it.
  return run_matmul(*ds, path, W_packed, ws, L, sx, s_w, M, N, K, y, y_dtype, acc_out, pdl,
                    pdl, stream, w_layout);
}

// Checks of one problem of a grouped call (the same rules as the forward).
bitnet_status check_problem(const bitnet_linear_problem& q) {
  bitnet_status st = check_shape(q.M, q.N, q.K);
  if (st != BITNET_OK) return st;
  if (q.w_layout != BITNET_LAYOUT_ROWS && q.w_layout != BITNET_LAYOUT_TILED)
    return BITNET_ERR_INVALID_ARG;
  if (q.M == 0) return BITNET_OK;
  if (!q.x || !q.W_packed || !q.s_w || !q.y || !ok_dtype(q.x_dtype) || !ok_dtype(q.y_dtype) ||
      !(q.eps >= 0.0f) || q.eps > 3.0e38f)
    return BITNET_ERR_INVALID_ARG;
  if (!aligned(q.x, 16) || (q.gamma && !aligned(q.gamma, 16)) || !aligned(q.W_packed, 16) ||
      !aligned(q.s_w, 4) || !aligned(q.y, 16))
    return BITNET_ERR_MISALIGNED;
  return BITNET_OK;
}

size_t grouped_workspace(int count, const bitnet_linear_problem* problems) {
  size_t total = 0;
  for (int i = 0; i < count; ++i) {
    const bitnet_linear_problem& q = problems[i];
    if (q.M > 0) total += fwd_layout(q.M, q.N, q.K).total;
  }
  return total;
}

// The launches of the decode problems of one grouped call.
struct DecodePlan {
  bool valid = false;
  int dev = -1;
  int count = 0;
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  bitnet_linear_problem probs[BITNET_MAX_GROUP];
  QuantLaunch QL;
  GemvLaunch GL;    // decode problems on row-major weights
  GtLaunch TL;      // decode problems on tiled weights
  long long G = 0;
  int n = 0;        // decode problems (both layouts)
  int nrow = 0;     // ... on row-major weights
  int qblocks = 0;  // blocks of the quant launch
  uint32_t stage = 0;
  // Larger problems (the tcgen05 kernel): quantized by the same grouped
  // launch, multiplied one after another.
  int nbig = 0;
  int big_src[BITNET_MAX_GROUP];
  uint8_t* big_q[BITNET_MAX_GROUP];       // workspace holding its quantized input
  FwdWorkspace big_qL[BITNET_MAX_GROUP];
  uint8_t* big_ws[BITNET_MAX_GROUP];      // its own workspace (split-K partials)
  FwdWorkspace big_L[BITNET_MAX_GROUP];
};

constexpr int kPlanCacheSize = 8;
thread_local DecodePlan g_plans[kPlanCacheSize];
thread_local int g_plan_next = 0;

bool same_problem(const bitnet_linear_problem& a, const bitnet_linear_problem& b) {
  return a.x == b.x && a.x_dtype == b.x_dtype && a.gamma == b.gamma &&
         std::memcmp(&a.eps, &b.eps, sizeof(float)) == 0 && a.W_packed == b.W_packed &&
         a.s_w == b.s_w && a.M == b.M && a.N == b.N && a.K == b.K && a.y == b.y &&
         a.y_dtype == b.y_dtype && a.w_layout == b.w_layout;
}

// Whether problems a and b quantize the same activations identically.
bool same_input(const bitnet_linear_problem& a, const bitnet_linear_problem& b) {
  return a.x == b.x && a.x_dtype == b.x_dtype && a.gamma == b.gamma &&
         std::memcmp(&a.eps, &b.eps, sizeof(float)) == 0 && a.M == b.M && a.K == b.K;
}

DecodePlan* cached_decode_plan(int count, const bitnet_linear_problem* problems, uint8_t* ws,
                               size_t ws_bytes) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  for (DecodePlan& p : g_plans) {
    if (!p.valid || p.dev != dev || p.count != count || p.ws != ws || p.ws_bytes != ws_bytes)
      continue;
    bool same = true;
    for (int i = 0; i < count && same; ++i) same = same_problem(p.probs[i], problems[i]);
    if (same) return &p;
  }
  return nullptr;
}

DecodePlan* new_decode_plan_slot(int count, const bitnet_linear_problem* problems, uint8_t* ws,
                                 size_t ws_bytes) {
  DecodePlan& p = g_plans[g_plan_next];
  g_plan_next = (g_plan_next + 1) % kPlanCacheSize;
  p.valid = false;
  if (cudaGetDevice(&p.dev) != cudaSuccess) p.dev = -1;
  p.count = count;
  p.ws = ws;
  p.ws_bytes = ws_bytes;
  for (int i = 0; i < count; ++i) p.probs[i] = problems[i];
  return &p;
}

// Plans the decode problems (M <= 16) of a grouped call: the matmul's work
// split, which partial regions the quant launch must clear, and one quant
// entry per distinct input (problems with the same x, dtype, gamma, eps, M
// and K share one quantization -- e.g. q/k/v or gate/up of one token batch).
bool build_decode_plan(const DeviceState& ds, int count, const bitnet_linear_problem* problems,
                       uint8_t* base, DecodePlan& plan) {
  QuantLaunch& QL = plan.QL;
  GemvLaunch& GL = plan.GL;
  GtLaunch& TL = plan.TL;
  QL = QuantLaunch{};
  GL.count = 0;
  TL.count = 0;
  // First pass: the matmul plans (the row-major one decides which partial
  // regions need zeroing by the quant launch).
  int nr = 0, nt = 0, mmax = 0;
  for (int i = 0; i < count; ++i) {
    const bitnet_linear_problem& q = problems[i];
    if (q.M == 0 || q.M > kGemvMaxM) continue;
    if (q.w_layout == BITNET_LAYOUT_TILED) {
      TL.prob[nt].M = static_cast<int>(q.M);
      TL.prob[nt].N = static_cast<int>(q.N);
      TL.prob[nt].K = static_cast<int>(q.K);
      ++nt;
      continue;
    }
    GL.prob[nr].M = static_cast<int>(q.M);
    GL.prob[nr].N = static_cast<int>(q.N);
    GL.prob[nr].K = static_cast<int>(q.K);
    mmax = std::max(mmax, static_cast<int>(q.M));
    ++nr;
  }
  GL.count = nr;
  TL.count = nt;
  plan.nrow = nr;
  plan.n = nr + nt;
  plan.G = nr > 0 ? plan_gemv_launch(GL, gemv_capacity(ds, mmax)) : 0;
  if (nt > 0) plan_gt_launch(TL, ds.num_sms);
  int qblocks = 0, qn = 0;
  uint32_t stage = 0;
  size_t off = 0;
  int src[BITNET_MAX_GROUP];            // problem index of each entry
  uint8_t* qws[BITNET_MAX_GROUP];       // its quantized-activation workspace
  FwdWorkspace qL[BITNET_MAX_GROUP];
  int kind[BITNET_MAX_GROUP];           // 0 row-major decode, 1 tiled decode, 2 tcgen05
  int n = 0, nb = 0;
  nr = 0;
  nt = 0;
  for (int i = 0; i < count; ++i) {
    const bitnet_linear_problem& q = problems[i];
    if (q.M == 0) continue;
    const FwdWorkspace L = fwd_layout(q.M, q.N, q.K);
    uint8_t* ws = base + off;
    off += L.total;
    const bool tiled = q.w_layout == BITNET_LAYOUT_TILED;
    const int kd = q.M > kGemvMaxM ? 2 : (tiled ? 1 : 0);
    // Region the quant launch clears: the tiled kernel's arrival counters,
    // the row-major kernel's split-K partials when its CTAs share rows, or
    // the tcgen05 kernel's split-K partials.
    const bool shared_rows = kd == 0 && gemv_problem_shared(GL, nr, plan.G);
    size_t zbytes = 0;
    void* zero = kd == 2 ? zero_region_for(ds, BITNET_PATH_GEMM, q.w_layout, q.M, q.N, q.K, ws,
                                           L, &zbytes)
                 : kd == 1 ? counter_region(ws, L, &zbytes)
                           : (shared_rows ? splitk_region(ws, L, &zbytes) : nullptr);
    int owner = -1;
    if (!shared_rows)
      for (int j = 0; j < n && owner < 0; ++j)
        if (kind[j] == kd && same_input(problems[src[j]], q)) owner = j;
    src[n] = i;
    kind[n] = kd;
    QuantProblem& qp = QL.prob[qn++];
    qp = QuantProblem{};
    qp.zero16 = static_cast<uint4*>(zero);
    qp.n_zero16 = zero ? static_cast<int64_t>(zbytes / 16) : 0;
    qp.zero_blocks = static_cast<int>(zero ? zero_blocks(zbytes) : 0);
    qp.block_begin = qblocks;
    if (owner >= 0) {
      // Reuse that problem's quantization; this entry only clears.
      qws[n] = qws[owner];
      qL[n] = qL[owner];
      qp.M = 0;
      if (!zero) --qn;
    } else {
      qws[n] = ws;
      qL[n] = L;
      qp.x = q.x;
      qp.gamma = q.gamma;
      qp.xi = reinterpret_cast<int8_t*>(ws + L.xq);
      qp.s_x = reinterpret_cast<float*>(ws + L.sx);
      qp.rowsum = reinterpret_cast<int32_t*>(ws + L.rs);
      qp.eps = q.eps;
      qp.M = static_cast<int>(q.M);
      qp.K = static_cast<int>(q.K);
      qp.x_bf16 = (q.x_dtype == BITNET_BF16) ? 1 : 0;
      qp.perm = kd == 2 ? 0 : 1;  // the decode matmuls' block order
      qp.tiled = kd == 1 ? 1 : 0;
      stage = std::max(stage, quant_stage_bytes(q.K, qp.x_bf16 != 0, q.gamma != nullptr));
    }
    if (owner < 0 || zero) qblocks += qp.M + qp.zero_blocks;
    const float* sx = reinterpret_cast<const float*>(qws[n] + qL[n].sx);
    if (kd == 2) {
      plan.big_src[nb] = i;
      plan.big_q[nb] = qws[n];
      plan.big_qL[nb] = qL[n];
      plan.big_ws[nb] = ws;
      plan.big_L[nb] = L;
      ++nb;
    } else if (tiled) {
      fill_gt_problem(TL.prob[nt], q.W_packed, qws[n], qL[n], ws, L, sx, q.s_w, q.M, q.N, q.K,
                      q.y, q.y_dtype, nullptr);
      ++nt;
    } else {
      if (!fill_gemv_problem(GL.maps[nr], GL.prob[nr], q.W_packed, qws[n], qL[n], ws, L, sx,
                             q.s_w, q.M, q.N, q.K, q.y, q.y_dtype, nullptr))
        return false;
      ++nr;
    }
    ++n;
  }
  QL.count = qn;
  plan.nbig = nb;
  plan.qblocks = qblocks;
  plan.stage = stage;
  plan.valid = true;
  return true;
}

bitnet_status forward_grouped_impl(int count, const bitnet_linear_problem* problems,
                                   void* workspace, size_t workspace_bytes, int phases,
                                   cudaStream_t stream) {
  if (count < 0 || count > BITNET_MAX_GROUP || (count > 0 && !problems))
    return BITNET_ERR_INVALID_ARG;
  if (phases < BITNET_PHASE_QUANTIZE || phases > BITNET_PHASE_ALL) return BITNET_ERR_INVALID_ARG;
  const bool do_quant = (phases & BITNET_PHASE_QUANTIZE) != 0;
  const bool do_matmul = (phases & BITNET_PHASE_MATMUL) != 0;
  for (int i = 0; i < count; ++i) {
    const bitnet_status st = check_problem(problems[i]);
    if (st != BITNET_OK) return st;
  }
  const size_t need = grouped_workspace(count, problems);
  if (need == 0) return BITNET_OK;
  if (!workspace || workspace_bytes < need) return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  uint8_t* base = static_cast<uint8_t*>(workspace);

  // Decode problems: one grouped quant launch, one grouped matmul launch,
  // planned once per distinct problem set (the plan is cached per thread).
  DecodePlan* plan = cached_decode_plan(count, problems, base, workspace_bytes);
  if (!plan) {
    plan = new_decode_plan_slot(count, problems, base, workspace_bytes);
    if (!build_decode_plan(*ds, count, problems, base, *plan)) {
      plan->valid = false;
      return BITNET_ERR_CUDA;
    }
  }
  {
    QuantLaunch& QL = plan->QL;
    GemvLaunch& GL = plan->GL;
    QL.trigger_dependents = do_matmul ? 1 : 0;
    if (do_quant && QL.count > 0) {
      QL.status = ds->status;
      QL.wait_limit_ns = kWaitLimitNs;
      const dim3 qg(static_cast<unsigned>(plan->qblocks));
      if (plan->stage <= kQuantStageMax)
        rmsnorm_quant_grouped_kernel<true><<<qg, kActThreads, plan->stage, stream>>>(QL);
      else
        rmsnorm_quant_grouped_kernel<false><<<qg, kActThreads, 0, stream>>>(QL);
      const bitnet_status st = launch_status();
      if (st != BITNET_OK) return st;
    }
    if (do_matmul && plan->nrow > 0) {
      // When the quant grid was just queued it started after every earlier
      // write to the weights, so the loads may begin before waiting on it.
      const bitnet_status st = launch_gemv_group(*ds, GL, plan->G, true, do_quant, stream);
      if (st != BITNET_OK) return st;
    }
    if (do_matmul && plan->TL.count > 0) {
      // Only a kernel of this library lets a dependent grid start early (the
      // quant grid above), and it writes no weights: the tiled kernel's
      // weight copies never need to wait.
      const bitnet_status st = launch_gt(*ds, plan->TL, true, stream);
      if (st != BITNET_OK) return st;
    }
  }
  if (!do_matmul) return BITNET_OK;
  // Larger problems: the tcgen05 kernel, one after another, on the inputs
  // the grouped launch quantized (each launch waits for the grid before it
  // -- which itself waited for the quant grid -- before reading them).
  for (int b = 0; b < plan->nbig; ++b) {
    const bitnet_linear_problem& q = problems[plan->big_src[b]];
    const uint8_t* qw = plan->big_q[b];
    const FwdWorkspace& qL = plan->big_qL[b];
    const bitnet_status st = launch_gemm(
        *ds, q.W_packed, reinterpret_cast<const int8_t*>(qw + qL.xq),
        reinterpret_cast<const int32_t*>(qw + qL.rs), reinterpret_cast<const float*>(qw + qL.sx),
        q.s_w, q.M, q.N, q.K, plan->big_ws[b], plan->big_L[b], q.y, q.y_dtype, nullptr, true,
        stream, q.w_layout == BITNET_LAYOUT_TILED);
    if (st != BITNET_OK) return st;
  }
  return BITNET_OK;
}

}  // namespace
}  // namespace bitnet

using namespace bitnet;

extern "C" {

BITNET_API const char* bitnet_status_string(int status) {
  switch (status) {
    case BITNET_OK: return "ok";
    case BITNET_ERR_INVALID_ARG: return "invalid argument";
    case BITNET_ERR_UNSUPPORTED_SHAPE:
      return "unsupported shape (need M <= 65535*128, 1 <= N <= 2^24, 64 <= K <= 2^20, "
             "K % 64 == 0)";
    case BITNET_ERR_MISALIGNED: return "misaligned pointer (tensors 16-byte, workspace 256-byte)";
    case BITNET_ERR_CUDA: return "CUDA error";
    case BITNET_ERR_TIMEOUT: return "bounded on-device wait timed out";
    case BITNET_ERR_WORKSPACE: return "workspace missing or too small";
    case BITNET_ERR_SCRATCH_LIMIT:
      return "N exceeds the static scratch of the allocation-free call (65536 rows)";
    default: return "unknown status";
  }
}

BITNET_API int bitnet_version(void) { return 200; }

BITNET_API int bitnet_last_cuda_error(const char** name) {
  const int e = g_last_cuda_error;
  g_last_cuda_error = 0;
  if (name) *name = cudaGetErrorName(static_cast<cudaError_t>(e));
  return e;
}

BITNET_API size_t bitnet_quantize_pack_weights_workspace_bytes(int64_t N, int64_t K) {
  (void)K;
  return N > 0 ? align256(8 * static_cast<size_t>(N)) : 0;
}

BITNET_API bitnet_status bitnet_quantize_pack_weights(const float* W, int64_t N, int64_t K,
                                                      uint8_t* W_packed, float* s_w,
                                                      void* workspace, size_t workspace_bytes,
                                                      bitnet_stream_t stream) {
  bitnet_status st = check_shape(0, N, K);
  if (st != BITNET_OK) return st;
  if (!W || !W_packed || !s_w) return BITNET_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(W_packed, 16) || !aligned(s_w, 4)) return BITNET_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < bitnet_quantize_pack_weights_workspace_bytes(N, K))
    return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  double* R = static_cast<double*>(workspace);
  row_abs_sum_kernel<<<static_cast<unsigned>(N), kWqThreads, 0, s>>>(W, K, R);
  abs_total_kernel<<<1, kWqThreads, 0, s>>>(R, N, K, s_w);
  const int64_t nwords = N * K / 16;
  const int64_t blocks = std::min<int64_t>((nwords + kWqThreads - 1) / kWqThreads,
                                           static_cast<int64_t>(ds->num_sms) * 16);
  pack_kernel<<<static_cast<unsigned>(blocks), kWqThreads, 0, s>>>(
      W, nwords, s_w, reinterpret_cast<uint32_t*>(W_packed));
  return launch_status();
}

BITNET_API bitnet_status bitnet_rmsnorm_quant_act(const void* x, int x_dtype, const float* gamma,
                                                  float eps, int64_t M, int64_t K, int8_t* x_q,
                                                  float* s_x, bitnet_stream_t stream) {
  bitnet_status st = check_shape(M, 1, K);
  if (st != BITNET_OK) return st;
  if (M == 0) return BITNET_OK;
  if (!x || !x_q || !s_x || !ok_dtype(x_dtype) || !(eps >= 0.0f) || eps > 3.0e38f)
    return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || (gamma && !aligned(gamma, 16)) || !aligned(x_q, 16) || !aligned(s_x, 4))
    return BITNET_ERR_MISALIGNED;
  if (!device_state()) return BITNET_ERR_CUDA;
  return launch_act_quant(x, x_dtype, gamma, eps, M, K, x_q, s_x, nullptr, kXNatural, false,
                          nullptr, 0, as_stream(stream));
}

BITNET_API size_t bitnet_linear_forward_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return 0;
  return fwd_layout(M, N, K).total;
}

BITNET_API bitnet_status bitnet_linear_forward(const void* x, int x_dtype, const float* gamma,
                                               float eps, const uint8_t* W_packed,
                                               const float* s_w, int64_t M, int64_t N, int64_t K,
                                               void* y, int y_dtype, void* workspace,
                                               size_t workspace_bytes, bitnet_stream_t stream) {
  if (!y && M != 0) return BITNET_ERR_INVALID_ARG;
  return forward_impl(x, x_dtype, gamma, eps, W_packed, s_w, M, N, K, y, y_dtype, workspace,
                      workspace_bytes, nullptr, nullptr, nullptr, BITNET_PATH_AUTO,
                      as_stream(stream));
}

BITNET_API bitnet_status bitnet_linear_quantize_input(const void* x, int x_dtype,
                                                      const float* gamma, float eps, int64_t M,
                                                      int64_t N, int64_t K, void* workspace,
                                                      size_t workspace_bytes,
                                                      bitnet_stream_t stream) {
  bitnet_status st = check_shape(M, N, K);
  if (st != BITNET_OK) return st;
  if (M == 0) return BITNET_OK;
  if (!x || !ok_dtype(x_dtype) || !(eps >= 0.0f) || eps > 3.0e38f) return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || (gamma && !aligned(gamma, 16))) return BITNET_ERR_MISALIGNED;
  const FwdWorkspace L = fwd_layout(M, N, K);
  if (!workspace || workspace_bytes < L.total) return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  if (!device_state()) return BITNET_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  size_t zbytes = 0;
  void* zero = (M <= kGemvMaxM) ? splitk_region(ws, L, &zbytes) : nullptr;
  const int path = resolve_path(BITNET_PATH_AUTO, M, N, K);  // the same as the matmul phase
  return launch_act_quant(x, x_dtype, gamma, eps, M, K, reinterpret_cast<int8_t*>(ws + L.xq),
                          reinterpret_cast<float*>(ws + L.sx),
                          reinterpret_cast<int32_t*>(ws + L.rs),
                          path == BITNET_PATH_GEMV ? kXDecode : kXInterleaved, M <= kGemvMaxM,
                          zero, zbytes, as_stream(stream));
}

BITNET_API bitnet_status bitnet_linear_matmul(const uint8_t* W_packed, const float* s_w,
                                              int64_t M, int64_t N, int64_t K, void* y,
                                              int y_dtype, void* workspace,
                                              size_t workspace_bytes, bitnet_stream_t stream) {
  bitnet_status st = check_shape(M, N, K);
  if (st != BITNET_OK) return st;
  if (M == 0) return BITNET_OK;
  if (!W_packed || !s_w || !y || !ok_dtype(y_dtype)) return BITNET_ERR_INVALID_ARG;
  if (!aligned(W_packed, 16) || !aligned(s_w, 4) || !aligned(y, 16)) return BITNET_ERR_MISALIGNED;
  const FwdWorkspace L = fwd_layout(M, N, K);
  if (!workspace || workspace_bytes < L.total) return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int path = resolve_path(BITNET_PATH_AUTO, M, N, K);
  return run_matmul(*ds, path, W_packed, ws, L, reinterpret_cast<const float*>(ws + L.sx), s_w,
                    M, N, K, y, y_dtype, nullptr, path == BITNET_PATH_GEMV, false,
                    as_stream(stream));
}

BITNET_API size_t bitnet_tiled_weights_bytes(int64_t N, int64_t K) {
  if (N < 1 || K < 64 || N > BITNET_MAX_N || K > BITNET_MAX_K || K % 64 != 0) return 0;
  return static_cast<size_t>(tiled_row_blocks(N) * tiled_chunks(K)) * kTileBytes;
}

BITNET_API bitnet_status bitnet_tile_weights(const uint8_t* W_packed, int64_t N, int64_t K,
                                             uint8_t* W_tiled, bitnet_stream_t stream) {
  bitnet_status st = check_shape(0, N, K);
  if (st != BITNET_OK) return st;
  if (!W_packed || !W_tiled) return BITNET_ERR_INVALID_ARG;
  if (!aligned(W_packed, 16) || !aligned(W_tiled, 16)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  const int64_t npieces = tiled_row_blocks(N) * tiled_chunks(K) * (kTileBytes / 16);
  const int64_t blocks = std::min<int64_t>((npieces + 255) / 256, 16LL * ds->num_sms);
  tile_weights_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(
      W_packed, N, K, W_tiled, npieces);
  return launch_status();
}

BITNET_API size_t bitnet_tiled_pair_weights_bytes(int64_t N, int64_t K) {
  return 2 * bitnet_tiled_weights_bytes(N, K);
}

BITNET_API bitnet_status bitnet_tile_weights_pair(const uint8_t* Wa_packed,
                                                  const uint8_t* Wb_packed, int64_t N, int64_t K,
                                                  uint8_t* W_pair, bitnet_stream_t stream) {
  bitnet_status st = check_shape(0, N, K);
  if (st != BITNET_OK) return st;
  if (!Wa_packed || !Wb_packed || !W_pair) return BITNET_ERR_INVALID_ARG;
  if (!aligned(Wa_packed, 16) || !aligned(Wb_packed, 16) || !aligned(W_pair, 16))
    return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  const int64_t npieces = tiled_row_blocks(N) * tiled_chunks(K) * (kTileBytes / 16);
  const int64_t blocks = std::min<int64_t>((npieces + 255) / 256, 16LL * ds->num_sms);
  tile_pair_weights_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(
      Wa_packed, Wb_packed, N, K, W_pair, npieces);
  return launch_status();
}

namespace {
// Workspace of the fused SwiGLU decode forward: the quantized input, its
// scales and row sums, partial slots of 256 table rows, the counters.
FwdWorkspace swiglu_layout(int64_t M, int64_t N, int64_t K) {
  FwdWorkspace w{};
  size_t o = 0;
  w.xq = o;
  o = align256(o + static_cast<size_t>(M * 256 * tiled_chunks(K)));
  w.sx = o;
  o = align256(o + 4 * static_cast<size_t>(M));
  w.rs = o;
  o = align256(o + 4 * static_cast<size_t>(M));
  const int64_t units = tiled_row_blocks(N) * tiled_chunks(K);
  w.acc = o;
  o = align256(o + 2 * static_cast<size_t>(std::min<int64_t>(kGtMaxCtas, units)) *
                       GtCfg<true, 1>::TAB_ROWS * 4 * static_cast<size_t>(M));
  w.cnt = o;
  o = align256(o + 4 * static_cast<size_t>(tiled_row_blocks(N)));
  w.total = o;
  return w;
}
}  // namespace

BITNET_API size_t bitnet_swiglu_forward_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return 0;
  return swiglu_layout(M, N, K).total;
}

BITNET_API bitnet_status bitnet_swiglu_forward(const void* x, int x_dtype, const float* gamma,
                                               float eps, const uint8_t* W_pair,
                                               const float* s_w_gate, const float* s_w_up,
                                               int64_t M, int64_t N, int64_t K, void* y,
                                               int y_dtype, void* workspace,
                                               size_t workspace_bytes, bitnet_stream_t stream) {
  bitnet_status st = check_shape(M, N, K);
  if (st != BITNET_OK) return st;
  if (M == 0) return BITNET_OK;
  if (M > kGemvMaxM) return BITNET_ERR_UNSUPPORTED_SHAPE;
  if (!x || !W_pair || !s_w_gate || !s_w_up || !y || !ok_dtype(x_dtype) || !ok_dtype(y_dtype) ||
      !(eps >= 0.0f) || eps > 3.0e38f)
    return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || (gamma && !aligned(gamma, 16)) || !aligned(W_pair, 16) ||
      !aligned(s_w_gate, 4) || !aligned(s_w_up, 4) || !aligned(y, 16))
    return BITNET_ERR_MISALIGNED;
  const FwdWorkspace L = swiglu_layout(M, N, K);
  if (!workspace || workspace_bytes < L.total) return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = as_stream(stream);
  size_t zbytes = 0;
  void* zero = counter_region(ws, L, &zbytes);
  float* sx = reinterpret_cast<float*>(ws + L.sx);
  st = launch_act_quant(x, x_dtype, gamma, eps, M, K, reinterpret_cast<int8_t*>(ws + L.xq), sx,
                        reinterpret_cast<int32_t*>(ws + L.rs), kXDecodeTiled, true, zero, zbytes,
                        s);
  if (st != BITNET_OK) return st;
  static thread_local GtLaunch GL;
  GL.count = 1;
  fill_gt_problem(GL.prob[0], W_pair, ws, L, ws, L, sx, s_w_gate, M, N, K, y, y_dtype, nullptr);
  GL.prob[0].s_w2 = s_w_up;
  plan_gt_launch(GL, ds->num_sms);
  return launch_gt(*ds, GL, true, s, true);
}

// ------------------------------------------------------ group-wise scales

namespace {

bitnet_status check_groups(int64_t K, int64_t group_k) {
  if (group_k < 256 || group_k % 256 != 0 || K % group_k != 0 || K / group_k > kGroupMaxG)
    return BITNET_ERR_UNSUPPORTED_SHAPE;
  return BITNET_OK;
}

struct GsWorkspace {
  size_t xq, sx, rs, gacc, part, cnt, total;
};

// x_q | s_x [M][G] | group row sums [M][G] | group sums [G][M][N] | tiled
// decode kernel's partial slots and counters (M <= 16).
GsWorkspace gs_layout(int64_t M, int64_t N, int64_t K, int64_t group_k) {
  GsWorkspace w{};
  const int64_t G = K / group_k;
  size_t o = 0;
  w.xq = o;
  o = align256(o + static_cast<size_t>(M * 256 * tiled_chunks(K)));
  w.sx = o;
  o = align256(o + 4 * static_cast<size_t>(M * G));
  w.rs = o;
  o = align256(o + 4 * static_cast<size_t>(M * G));
  w.gacc = o;
  o = align256(o + 4 * static_cast<size_t>(G * M * N));
  const int64_t tiles = tiled_row_blocks(N) * tiled_chunks(K);
  w.part = o;
  if (M <= kGemvMaxM)
    o = align256(o + 2 * static_cast<size_t>(std::min<int64_t>(kGtMaxCtas, tiles)) *
                         kTileRows * 4 * static_cast<size_t>(M));
  w.cnt = o;
  if (M <= kGemvMaxM) o = align256(o + 4 * static_cast<size_t>(tiled_row_blocks(N) * G));
  w.total = o;
  return w;
}

}  // namespace

BITNET_API size_t bitnet_quantize_pack_weights_group_scales_workspace_bytes(int64_t N,
                                                                            int64_t K,
                                                                            int64_t group_k) {
  if (N <= 0 || K <= 0 || group_k <= 0 || K % group_k != 0) return 0;
  return align256(8 * static_cast<size_t>(N * (K / group_k)));
}

BITNET_API bitnet_status bitnet_quantize_pack_weights_group_scales(
    const float* W, int64_t N, int64_t K, int64_t group_k, uint8_t* W_packed, float* s_w,
    void* workspace, size_t workspace_bytes, bitnet_stream_t stream) {
  bitnet_status st = check_shape(0, N, K);
  if (st != BITNET_OK) return st;
  st = check_groups(K, group_k);
  if (st != BITNET_OK) return st;
  if (!W || !W_packed || !s_w) return BITNET_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(W_packed, 16) || !aligned(s_w, 4)) return BITNET_ERR_MISALIGNED;
  if (!workspace ||
      workspace_bytes < bitnet_quantize_pack_weights_group_scales_workspace_bytes(N, K, group_k))
    return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  const int64_t G = K / group_k;
  double* R = static_cast<double*>(workspace);
  group_row_abs_sum_kernel<<<static_cast<unsigned>(N), kWqThreads, 0, s>>>(W, K, group_k, R);
  group_abs_total_kernel<<<static_cast<unsigned>(G), kWqThreads, 0, s>>>(R, N, G, group_k, s_w);
  const int64_t nwords = N * K / 16;
  const int64_t blocks = std::min<int64_t>((nwords + kWqThreads - 1) / kWqThreads,
                                           static_cast<int64_t>(ds->num_sms) * 16);
  group_pack_kernel<<<static_cast<unsigned>(blocks), kWqThreads, 0, s>>>(
      W, nwords, K, group_k, s_w, reinterpret_cast<uint32_t*>(W_packed));
  return launch_status();
}

BITNET_API size_t bitnet_linear_forward_group_scales_workspace_bytes(int64_t M, int64_t N,
                                                                     int64_t K,
                                                                     int64_t group_k) {
  if (M < 0 || N < 0 || K <= 0 || group_k <= 0 || K % group_k != 0) return 0;
  return gs_layout(M, N, K, group_k).total;
}

BITNET_API bitnet_status bitnet_linear_forward_group_scales(
    const void* x, int x_dtype, const float* gamma, float eps, const uint8_t* W_packed,
    int w_layout, const float* s_w, int64_t M, int64_t N, int64_t K, int64_t group_k, void* y,
    int y_dtype, void* workspace, size_t workspace_bytes, int8_t* x_q_out, float* s_x_out,
    int32_t* acc_out, bitnet_stream_t stream) {
  bitnet_status st = check_shape(M, N, K);
  if (st != BITNET_OK) return st;
  st = check_groups(K, group_k);
  if (st != BITNET_OK) return st;
  if (M == 0) return BITNET_OK;
  if (!x || !W_packed || !s_w || (!y && !acc_out) || !ok_dtype(x_dtype) || !(eps >= 0.0f) ||
      eps > 3.0e38f || (y && !ok_dtype(y_dtype)))
    return BITNET_ERR_INVALID_ARG;
  if (w_layout != BITNET_LAYOUT_ROWS && w_layout != BITNET_LAYOUT_TILED)
    return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || (gamma && !aligned(gamma, 16)) || !aligned(W_packed, 16) ||
      !aligned(s_w, 4) || (y && !aligned(y, 16)) || (x_q_out && !aligned(x_q_out, 16)) ||
      (s_x_out && !aligned(s_x_out, 4)) || (acc_out && !aligned(acc_out, 16)))
    return BITNET_ERR_MISALIGNED;
  const GsWorkspace L = gs_layout(M, N, K, group_k);
  if (!workspace || workspace_bytes < L.total) return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int64_t G = K / group_k;
  const bool tiled_decode = w_layout == BITNET_LAYOUT_TILED && M <= kGemvMaxM;
  int8_t* xq = reinterpret_cast<int8_t*>(ws + L.xq);
  float* sx = reinterpret_cast<float*>(ws + L.sx);
  int32_t* rs = reinterpret_cast<int32_t*>(ws + L.rs);
  int32_t* gacc = acc_out ? acc_out : reinterpret_cast<int32_t*>(ws + L.gacc);
  const bool bf16 = x_dtype == BITNET_BF16;
  if (x_q_out || s_x_out) {   // debug export: natural order, same arithmetic
    float* sx_dbg = s_x_out ? s_x_out : sx;
    int8_t* xq_dbg = x_q_out ? x_q_out : xq;
    if (bf16)
      group_rmsnorm_quant_kernel<true><<<static_cast<unsigned>(M), kActThreads, 0, s>>>(
          x, gamma, eps, M, K, group_k, xq_dbg, sx_dbg, nullptr, 0, 0, 1, nullptr, 0, 0);
    else
      group_rmsnorm_quant_kernel<false><<<static_cast<unsigned>(M), kActThreads, 0, s>>>(
          x, gamma, eps, M, K, group_k, xq_dbg, sx_dbg, nullptr, 0, 0, 1, nullptr, 0, 0);
    st = launch_status();
    if (st != BITNET_OK) return st;
  }
  size_t zbytes = tiled_decode ? L.total - L.cnt : 0;
  uint4* zero = zbytes ? reinterpret_cast<uint4*>(ws + L.cnt) : nullptr;
  const int64_t zb = zero ? zero_blocks(zbytes) : 0;
  const dim3 qgrid(static_cast<unsigned>(M + zb));
  if (bf16)
    group_rmsnorm_quant_kernel<true><<<qgrid, kActThreads, 0, s>>>(
        x, gamma, eps, M, K, group_k, xq, sx, rs, tiled_decode ? 1 : 0, tiled_decode ? 1 : 0, 0,
        zero, zero ? static_cast<int64_t>(zbytes / 16) : 0, 1);
  else
    group_rmsnorm_quant_kernel<false><<<qgrid, kActThreads, 0, s>>>(
        x, gamma, eps, M, K, group_k, xq, sx, rs, tiled_decode ? 1 : 0, tiled_decode ? 1 : 0, 0,
        zero, zero ? static_cast<int64_t>(zbytes / 16) : 0, 1);
  st = launch_status();
  if (st != BITNET_OK) return st;
  if (tiled_decode) {
    static thread_local GtLaunch GL;
    GL.count = 1;
    GtProblem& q = GL.prob[0];
    FwdWorkspace FL{};
    FL.xq = L.xq;
    FL.sx = L.sx;
    FL.rs = L.rs;
    FL.acc = L.part;
    FL.cnt = L.cnt;
    FL.total = L.total;
    fill_gt_problem(q, W_packed, ws, FL, ws, FL, sx, s_w, M, N, K, nullptr, BITNET_F32, nullptr);
    q.gc = static_cast<int>(group_k / 256);
    q.G = static_cast<int>(G);
    q.gacc = gacc;
    plan_gt_launch(GL, ds->num_sms);
    st = launch_gt(*ds, GL, true, s);
  } else {
    // tcgen05: one K split per group, each CTA writes its group's sums
    GemmPlan pl = plan_gemm(M, N, K, ds->num_sms);
    pl.steps_per_split = static_cast<int>(group_k / 256);
    pl.ksplit = static_cast<int>(G);
    st = launch_gemm_groups(*ds, W_packed, xq, rs, M, N, K, G, gacc, pl,
                            w_layout == BITNET_LAYOUT_TILED, s);
  }
  if (st != BITNET_OK) return st;
  if (y) {
    const int64_t blocks = std::min<int64_t>((M * N + 255) / 256, 16LL * ds->num_sms);
    group_combine_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        gacc, sx, s_w, M, N, G, y, y_dtype == BITNET_BF16 ? 1 : 0);
    st = launch_status();
  }
  return st;
}

BITNET_API bitnet_status bitnet_linear_forward_ex(const bitnet_linear_problem* problem,
                                                  void* workspace, size_t workspace_bytes,
                                                  int8_t* x_q_out, float* s_x_out,
                                                  int32_t* acc_out, int path,
                                                  bitnet_stream_t stream) {
  if (!problem) return BITNET_ERR_INVALID_ARG;
  const bitnet_linear_problem& q = *problem;
  if (!q.y && !acc_out && q.M != 0) return BITNET_ERR_INVALID_ARG;
  return forward_impl(q.x, q.x_dtype, q.gamma, q.eps, q.W_packed, q.s_w, q.M, q.N, q.K, q.y,
                      q.y_dtype, workspace, workspace_bytes, x_q_out, s_x_out, acc_out, path,
                      as_stream(stream), q.w_layout);
}

BITNET_API size_t bitnet_linear_forward_grouped_workspace_bytes(
    int count, const bitnet_linear_problem* problems) {
  if (count < 0 || count > BITNET_MAX_GROUP || (count > 0 && !problems)) return 0;
  for (int i = 0; i < count; ++i)
    if (problems[i].M < 0 || problems[i].N < 0 || problems[i].K < 0) return 0;
  return grouped_workspace(count, problems);
}

BITNET_API bitnet_status bitnet_linear_forward_grouped(int count,
                                                       const bitnet_linear_problem* problems,
                                                       void* workspace, size_t workspace_bytes,
                                                       int phases, bitnet_stream_t stream) {
  return forward_grouped_impl(count, problems, workspace, workspace_bytes, phases,
                              as_stream(stream));
}

BITNET_API bitnet_status bitnet_linear_forward_debug(
    const void* x, int x_dtype, const float* gamma, float eps, const uint8_t* W_packed,
    const float* s_w, int64_t M, int64_t N, int64_t K, void* y, int y_dtype, void* workspace,
    size_t workspace_bytes, int8_t* x_q_out, float* s_x_out, int32_t* acc_out, int path,
    bitnet_stream_t stream) {
  return forward_impl(x, x_dtype, gamma, eps, W_packed, s_w, M, N, K, y, y_dtype, workspace,
                      workspace_bytes, x_q_out, s_x_out, acc_out, path, as_stream(stream));
}

BITNET_API bitnet_status bitnet_ternary_matmul_i32(const int8_t* x_q, const uint8_t* W_packed,
                                                   int64_t M, int64_t N, int64_t K, int32_t* acc,
                                                   void* workspace, size_t workspace_bytes,
                                                   int path, bitnet_stream_t stream) {
  bitnet_status st = check_shape(M, N, K);
  if (st != BITNET_OK) return st;
  if (M == 0) return BITNET_OK;
  if (!x_q || !W_packed || !acc) return BITNET_ERR_INVALID_ARG;
  if (path < BITNET_PATH_AUTO || path > BITNET_PATH_GEMM) return BITNET_ERR_INVALID_ARG;
  path = resolve_path(path, M, N, K);
  if (path == BITNET_PATH_GEMV && M > kGemvMaxM) return BITNET_ERR_INVALID_ARG;
  if (!aligned(x_q, 16) || !aligned(W_packed, 16) || !aligned(acc, 16))
    return BITNET_ERR_MISALIGNED;
  const FwdWorkspace L = fwd_layout(M, N, K);
  if (!workspace || workspace_bytes < L.total) return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  size_t zbytes = 0;
  void* zero = needs_zeroed_partials(*ds, path, M, N, K) ? splitk_region(ws, L, &zbytes)
                                                          : nullptr;
  const int64_t zb = zero ? zero_blocks(zbytes) : 0;
  interleave_rowsum_kernel<<<static_cast<unsigned>(M + zb), kActThreads, 0, s>>>(
      x_q, M, K, reinterpret_cast<int8_t*>(ws + L.xq), reinterpret_cast<int32_t*>(ws + L.rs),
      static_cast<uint4*>(zero), zero ? static_cast<int64_t>(zbytes / 16) : 0,
      path == BITNET_PATH_GEMV ? 1 : 0);
  st = launch_status();
  if (st != BITNET_OK) return st;
  return run_matmul(*ds, path, W_packed, ws, L, nullptr, nullptr, M, N, K, nullptr, BITNET_F32,
                    acc, false, false, s);
}

BITNET_API size_t bitnet_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return bitnet_linear_forward_workspace_bytes(M, N, K);
}

BITNET_API bitnet_status bitnet_last_device_status(bitnet_stream_t stream) {
  return bitnet_device_status(stream, 0, nullptr);
}

BITNET_API bitnet_status bitnet_device_status(bitnet_stream_t stream, int reset, int* detail) {
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, ds->status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return BITNET_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BITNET_ERR_CUDA;
  if (detail) *detail = v;
  if (reset && v != 0) {
    if (cudaMemsetAsync(ds->status, 0, sizeof(int), s) != cudaSuccess) return BITNET_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return BITNET_ERR_CUDA;
  }
  return v == 0 ? BITNET_OK : BITNET_ERR_TIMEOUT;
}

// ------------------------------------------------ lambda-warmup fake quant

}  // extern "C"

namespace {

// 2-D bf16 tensor [rows][inner] (row stride in bytes), boxes of 64 x
// box_rows elements, 128-byte swizzle (the tcgen05 K-major canonical layout);
// out-of-range elements read as zero.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t row_stride, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int BN>
bitnet_status launch_wg_bn(const CUtensorMap& ta, const CUtensorMap& tb, const WgParams& p,
                           cudaStream_t s) {
  static std::once_flag once;
  static bool ok = false;
  std::call_once(once, []() {
    ok = cudaFuncSetAttribute(bf16_gemm_nt_kernel<BN>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              WgCfg<BN>::SMEM_DYN) == cudaSuccess;
  });
  if (!ok) return BITNET_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>((p.N + 127) / 128),
                  static_cast<unsigned>((p.M + BN - 1) / BN));
  bf16_gemm_nt_kernel<BN><<<grid, WgCfg<BN>::THREADS, WgCfg<BN>::SMEM_DYN, s>>>(ta, tb, p);
  return launch_status();
}

// y[m][n] (row stride ldy) = sum_k B[m][k] A[n][k]; A [N][K], B [M][K] bf16
// with row strides lda, ldb elements (multiples of 8).
bitnet_status launch_bf16_gemm_nt(const DeviceState& ds, const void* A, int64_t lda,
                                  const void* B, int64_t ldb, int64_t M, int64_t N, int64_t K,
                                  void* y, int64_t ldy, int y_dtype, cudaStream_t s) {
  if (M == 0 || N == 0) return BITNET_OK;
  const int BN = M <= 64 ? 64 : (M <= 128 ? 128 : 256);
  CUtensorMap ta, tb;
  if (!make_tmap_bf16(&ta, A, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                      static_cast<uint64_t>(2 * lda), 128) ||
      !make_tmap_bf16(&tb, B, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                      static_cast<uint64_t>(2 * ldb), static_cast<uint32_t>(BN)))
    return BITNET_ERR_CUDA;
  WgParams p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.y = y;
  p.ldy = ldy;
  p.y_bf16 = y_dtype == BITNET_BF16 ? 1 : 0;
  p.status = ds.status;
  p.wait_limit_ns = kWaitLimitNs;
  p.use_pdl = 0;
  if (BN == 64) return launch_wg_bn<64>(ta, tb, p, s);
  if (BN == 128) return launch_wg_bn<128>(ta, tb, p, s);
  return launch_wg_bn<256>(ta, tb, p, s);
}

bitnet_status check_warmup_shape(int64_t M, int64_t N, int64_t K, float lambda) {
  if (M < 0 || N < 0 || K < 0 || !(lambda >= 0.0f) || lambda > 1.0f)
    return BITNET_ERR_INVALID_ARG;
  if (N < 1 || K < 8 || K % 8 != 0 || N % 8 != 0 || N > BITNET_MAX_N || K > BITNET_MAX_K ||
      M > BITNET_MAX_M)
    return BITNET_ERR_UNSUPPORTED_SHAPE;
  return BITNET_OK;
}

int64_t round8(int64_t v) { return (v + 7) / 8 * 8; }

}  // namespace

extern "C" {

BITNET_API size_t bitnet_warmup_quantize_weights_workspace_bytes(int64_t N, int64_t K) {
  return bitnet_quantize_pack_weights_workspace_bytes(N, K);
}

BITNET_API bitnet_status bitnet_warmup_quantize_weights(const float* W, int64_t N, int64_t K,
                                                        float lambda, void* W_lam, float* s_w,
                                                        void* workspace, size_t workspace_bytes,
                                                        bitnet_stream_t stream) {
  bitnet_status st = check_warmup_shape(0, N, K, lambda);
  if (st != BITNET_OK) return st;
  if (!W || !W_lam || !s_w) return BITNET_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(W_lam, 16) || !aligned(s_w, 4)) return BITNET_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < bitnet_warmup_quantize_weights_workspace_bytes(N, K))
    return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  double* R = static_cast<double*>(workspace);
  row_abs_sum_kernel<<<static_cast<unsigned>(N), kWqThreads, 0, s>>>(W, K, R);
  abs_total_kernel<<<1, kWqThreads, 0, s>>>(R, N, K, s_w);
  const int64_t n4 = N * K / 4;
  const int64_t blocks = std::min<int64_t>((n4 + 255) / 256, 16LL * ds->num_sms);
  warmup_weights_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      W, n4, s_w, lambda, static_cast<__nv_bfloat16*>(W_lam));
  return launch_status();
}

BITNET_API size_t bitnet_warmup_forward_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  (void)N;
  if (M < 0 || K < 0) return 0;
  return align256(2 * static_cast<size_t>(M * K));
}

BITNET_API bitnet_status bitnet_warmup_forward(const void* x, int x_dtype, const float* gamma,
                                               float eps, const void* W_lam, int64_t M,
                                               int64_t N, int64_t K, float lambda, void* y,
                                               int y_dtype, void* x_lam, void* workspace,
                                               size_t workspace_bytes, bitnet_stream_t stream) {
  bitnet_status st = check_warmup_shape(M, N, K, lambda);
  if (st != BITNET_OK) return st;
  if (M == 0) return BITNET_OK;
  if (!x || !W_lam || !y || !ok_dtype(x_dtype) || !ok_dtype(y_dtype) || !(eps >= 0.0f) ||
      eps > 3.0e38f)
    return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || (gamma && !aligned(gamma, 16)) || !aligned(W_lam, 16) ||
      !aligned(y, 4) || (x_lam && !aligned(x_lam, 16)))
    return BITNET_ERR_MISALIGNED;
  if (!x_lam && (!workspace || workspace_bytes < bitnet_warmup_forward_workspace_bytes(M, N, K)))
    return BITNET_ERR_WORKSPACE;
  if (!x_lam && !aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  __nv_bfloat16* xl = static_cast<__nv_bfloat16*>(x_lam ? x_lam : workspace);
  if (x_dtype == BITNET_BF16)
    warmup_act_kernel<true><<<static_cast<unsigned>(M), kActThreads, 0, s>>>(x, gamma, eps, K,
                                                                             lambda, xl);
  else
    warmup_act_kernel<false><<<static_cast<unsigned>(M), kActThreads, 0, s>>>(x, gamma, eps, K,
                                                                              lambda, xl);
  st = launch_status();
  if (st != BITNET_OK) return st;
  return launch_bf16_gemm_nt(*ds, W_lam, K, xl, K, M, N, K, y, N, y_dtype, s);
}

BITNET_API size_t bitnet_warmup_backward_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return 0;
  const int64_t Mp = round8(M);
  return align256(2 * static_cast<size_t>(K * N)) + align256(2 * static_cast<size_t>(N * Mp)) +
         align256(2 * static_cast<size_t>(K * Mp));
}

BITNET_API bitnet_status bitnet_warmup_backward(const void* dy, const void* x_lam,
                                                const void* W_lam, int64_t M, int64_t N,
                                                int64_t K, float* dx, float* dW, void* workspace,
                                                size_t workspace_bytes, bitnet_stream_t stream) {
  bitnet_status st = check_warmup_shape(M, N, K, 0.0f);
  if (st != BITNET_OK) return st;
  if (!dy || (dx && !W_lam) || (dW && !x_lam)) return BITNET_ERR_INVALID_ARG;
  if (!aligned(dy, 16) || (x_lam && !aligned(x_lam, 16)) || (W_lam && !aligned(W_lam, 16)) ||
      (dx && !aligned(dx, 4)) || (dW && !aligned(dW, 4)))
    return BITNET_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < bitnet_warmup_backward_workspace_bytes(M, N, K))
    return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  if (dW && M == 0) {
    if (cudaMemsetAsync(dW, 0, 4 * static_cast<size_t>(N * K), s) != cudaSuccess)
      return BITNET_ERR_CUDA;
  }
  if (M == 0) return BITNET_OK;
  const int64_t Mp = round8(M);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  __nv_bfloat16* WT = reinterpret_cast<__nv_bfloat16*>(ws);                    // [K][N]
  uint8_t* p1 = ws + align256(2 * static_cast<size_t>(K * N));
  __nv_bfloat16* dyT = reinterpret_cast<__nv_bfloat16*>(p1);                   // [N][Mp]
  __nv_bfloat16* xT = reinterpret_cast<__nv_bfloat16*>(p1 + align256(2 * static_cast<size_t>(N * Mp)));  // [K][Mp]
  const __nv_bfloat16* dyb = static_cast<const __nv_bfloat16*>(dy);
  auto transpose = [&](const __nv_bfloat16* src, int64_t R, int64_t C, __nv_bfloat16* dst,
                       int64_t ldd) {
    const dim3 grid(static_cast<unsigned>((C + 31) / 32), static_cast<unsigned>((ldd + 31) / 32));
    transpose_bf16_kernel<<<grid, 256, 0, s>>>(src, R, C, dst, ldd);
    return launch_status();
  };
  if (dx) {
    // dx [M][K] = dy [M][N] . W_lam [N][K]: B = dy (K-major over n), A = W_lam^T.
    st = transpose(static_cast<const __nv_bfloat16*>(W_lam), N, K, WT, N);
    if (st != BITNET_OK) return st;
    st = launch_bf16_gemm_nt(*ds, WT, N, dyb, N, M, K, N, dx, K, BITNET_F32, s);
    if (st != BITNET_OK) return st;
  }
  if (dW) {
    // dW [N][K] = dy^T [N][M] . x_lam [M][K]: B = dy^T, A = x_lam^T (zero-padded to Mp).
    st = transpose(dyb, M, N, dyT, Mp);
    if (st != BITNET_OK) return st;
    st = transpose(static_cast<const __nv_bfloat16*>(x_lam), M, K, xT, Mp);
    if (st != BITNET_OK) return st;
    st = launch_bf16_gemm_nt(*ds, xT, Mp, dyT, Mp, N, K, Mp, dW, K, BITNET_F32, s);
    if (st != BITNET_OK) return st;
  }
  return BITNET_OK;
}

// ------------------------------------------------------ BitDelta 1-bit deltas

BITNET_API size_t bitnet_bitdelta_compress_workspace_bytes(int64_t N, int64_t K) {
  (void)K;
  return N > 0 ? align256(8 * static_cast<size_t>(N)) : 0;
}

BITNET_API bitnet_status bitnet_bitdelta_compress(const void* W_base, const void* W_fine,
                                                  int64_t N, int64_t K, uint32_t* signs,
                                                  float* alpha, void* workspace,
                                                  size_t workspace_bytes,
                                                  bitnet_stream_t stream) {
  if (N < 0 || K < 0) return BITNET_ERR_INVALID_ARG;
  if (N < 1 || K < 32 || K % 32 != 0 || N > BITNET_MAX_N || K > BITNET_MAX_K)
    return BITNET_ERR_UNSUPPORTED_SHAPE;
  if (!W_base || !W_fine || !signs || !alpha) return BITNET_ERR_INVALID_ARG;
  if (!aligned(W_base, 16) || !aligned(W_fine, 16) || !aligned(signs, 4) || !aligned(alpha, 4))
    return BITNET_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < bitnet_bitdelta_compress_workspace_bytes(N, K))
    return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_MISALIGNED;
  if (!device_state()) return BITNET_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  double* R = static_cast<double*>(workspace);
  bitdelta_row_kernel<<<static_cast<unsigned>(N), kWqThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(W_base), static_cast<const __nv_bfloat16*>(W_fine), K,
      signs, R);
  bitdelta_alpha_kernel<<<1, kWqThreads, 0, s>>>(R, N, K, alpha);
  return launch_status();
}

BITNET_API bitnet_status bitnet_bitdelta_forward(const void* x, const void* W_base,
                                                 const uint32_t* signs, const float* alpha,
                                                 int64_t B, int64_t N, int64_t K, void* y,
                                                 int y_dtype, bitnet_stream_t stream) {
  if (B < 0 || N < 0 || K < 0) return BITNET_ERR_INVALID_ARG;
  if (B > kBdMaxTenants || N < 1 || K < 32 || K % 32 != 0 || N > BITNET_MAX_N ||
      K > BITNET_MAX_K || (N + 15) / 16 > 0x7FFFFFFFLL)
    return BITNET_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return BITNET_OK;
  if (!x || !W_base || !signs || !alpha || !y || !ok_dtype(y_dtype)) return BITNET_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(W_base, 16) || !aligned(signs, 4) || !aligned(alpha, 4) ||
      !aligned(y, 4))
    return BITNET_ERR_MISALIGNED;
  if (!device_state()) return BITNET_ERR_CUDA;
  bitdelta_forward_kernel<<<static_cast<unsigned>((N + 15) / 16), 32 * kBdWarps, 0,
                            as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(W_base), signs,
      alpha, static_cast<int>(B), N, K, y, y_dtype == BITNET_BF16 ? 1 : 0);
  return launch_status();
}

}  // extern "C"

namespace bitnet {
namespace {
__global__ void bounded_wait_selftest_kernel(int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // nothing ever arrives on it
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0u, nullptr, limit_ns))
    record_failure(status, DEV_TIMEOUT_SELFTEST);
}
}  // namespace
}  // namespace bitnet

namespace bitnet {
namespace {
__global__ void divide_selftest_kernel(const float* __restrict__ a, const float* __restrict__ b,
                                       float* __restrict__ q, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
  {
    // The epilogue's division for numerators it can see (integer-valued or
    // not, |a| in {0} U [1, 2^31]); any other numerator takes the IEEE
    // division, so the result is always RN(a / b).
    const float av = fabsf(a[i]);
    const bool in_range = a[i] == 0.0f || (av >= 1.0f && av <= 0x1p31f);
    q[i] = in_range ? div_rn_int(a[i], b[i], recip_for_div(b[i])) : __fdiv_rn(a[i], b[i]);
  }
}
}  // namespace
}  // namespace bitnet

extern "C" BITNET_API bitnet_status bitnet_selftest_divide(const float* a, const float* b,
                                                           float* q, int64_t n,
                                                           bitnet_stream_t stream) {
  if (n < 0 || (n > 0 && (!a || !b || !q))) return BITNET_ERR_INVALID_ARG;
  if (n == 0) return BITNET_OK;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(q, 16)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 4 * ds->num_sms);
  divide_selftest_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(a, b, q,
                                                                                        n);
  return launch_status();
}

extern "C" BITNET_API bitnet_status bitnet_selftest_mma_i8(int64_t iters, int ctas, int a_in_tmem,
                                                          bitnet_stream_t stream) {
  if (iters < 1 || iters > 100000000LL || ctas < 1 || ctas > 65535) return BITNET_ERR_INVALID_ARG;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  if (a_in_tmem)
    mma_i8_peak_kernel<true><<<ctas, 128, kPeakSmem, as_stream(stream)>>>(iters, ds->status,
                                                                          kWaitLimitNs);
  else
    mma_i8_peak_kernel<false><<<ctas, 128, kPeakSmem, as_stream(stream)>>>(iters, ds->status,
                                                                           kWaitLimitNs);
  return launch_status();
}

extern "C" BITNET_API bitnet_status bitnet_selftest_bounded_wait(uint64_t limit_ns,
                                                                 bitnet_stream_t stream) {
  if (limit_ns < 1000ull || limit_ns > 1000000000ull) return BITNET_ERR_INVALID_ARG;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  bounded_wait_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>(ds->status, limit_ns);
  return launch_status();
}

// ---------------------------------------------------------------------------
// Allocation-free weight quantization: the fp64 per-row |W| sums live in a
// file-scope device array instead of a caller workspace, for callers that
// cannot allocate device memory.  The array is per device (one copy in every
// context that loads this library) and lives until the process exits.

namespace bitnet {
namespace {

static __device__ __align__(256) double g_static_row_sums[BITNET_STATIC_SCRATCH_MAX_N];

struct StaticScratch {
  std::once_flag once;
  double* ptr = nullptr;  // device address of g_static_row_sums on this device
};
StaticScratch g_static_scratch[kMaxDevices];

// In host code the array's name is only a host-side handle; the kernels need
// its device address, looked up once per device with that device current.
double* static_row_sums() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  StaticScratch& sc = g_static_scratch[dev];
  std::call_once(sc.once, [&sc]() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_row_sums) == cudaSuccess)
      sc.ptr = static_cast<double*>(p);
  });
  return sc.ptr;
}

}  // namespace
}  // namespace bitnet

extern "C" BITNET_API bitnet_status bitnet_quantize_pack_weights_static(
    const float* W, int64_t N, int64_t K, uint8_t* W_packed, float* s_w,
    bitnet_stream_t stream) {
  bitnet_status st = check_shape(0, N, K);
  if (st != BITNET_OK) return st;
  if (N > BITNET_STATIC_SCRATCH_MAX_N) return BITNET_ERR_SCRATCH_LIMIT;
  if (!W || !W_packed || !s_w) return BITNET_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(W_packed, 16) || !aligned(s_w, 4)) return BITNET_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (!ds) return BITNET_ERR_CUDA;
  double* R = static_row_sums();
  if (!R) return BITNET_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  row_abs_sum_kernel<<<static_cast<unsigned>(N), kWqThreads, 0, s>>>(W, K, R);
  abs_total_kernel<<<1, kWqThreads, 0, s>>>(R, N, K, s_w);
  const int64_t nwords = N * K / 16;
  const int64_t blocks = std::min<int64_t>((nwords + kWqThreads - 1) / kWqThreads,
                                           static_cast<int64_t>(ds->num_sms) * 16);
  pack_kernel<<<static_cast<unsigned>(blocks), kWqThreads, 0, s>>>(
      W, nwords, s_w, reinterpret_cast<uint32_t*>(W_packed));
  return launch_status();
}
