/*
 * bitnet_b200.h -- C ABI of the B200 (sm_100a) BitNet b1.58 BitLinear forward.
 *
 * The forward pass, as the pages define it:
 *   1. RMSNorm of each token row, then per-token absmax quantization of the
 *      activations to int8 in [-128, 127]
 *      ("LLM を 1.58 ビットにファインチューニング：BitNet による極端な量子化",
 *       section 量子化の仕組み, activations bullet; "[論文レビュー] The Era of
 *       1-bit LLMs", section 提案手法, RMSNorm);
 *   2. ternary weights from a per-tensor absmean scale, four 2-bit codes per
 *      byte (same first page, 量子化の仕組み weights bullet and 主な発見
 *      packing; The Era of 1-bit LLMs review, 提案手法 absmean);
 *   3. an integer matmul with int32 accumulation (first page, 計算パラダイム);
 *   4. the rescale y = acc / (s_x * s_w) (first page, 量子化の仕組み; the
 *      bitnet.cpp article, section 数学的基礎 item 3).
 *
 * Exact arithmetic of every step (all of it reproduced bit for bit by the
 * kernels):
 *   r      = 1 / sqrt(ss / K + eps), ss = sum of x^2 over the row, reduced in a
 *            fixed order: element k goes to partial (k/8) mod 256 (fp32,
 *            fused multiply-add, increasing k), then partial i absorbs
 *            partial i+s for s = 128, 64, ..., 1; division and sqrt correctly
 *            rounded.  A row with ss/K + eps == 0 normalises to all zeros.
 *   x_n    = (x * r) * gamma                  (two rounded fp32 products)
 *   s_x    = 127 / max(max|x_n|, 1e-5)
 *   x_q    = clamp(rint(x_n * s_x), -128, 127)          (ties to even)
 *   S      = sum |W| in fp64: per row, element k to partial (k/4) mod 256,
 *            same tree; then row sums to partial n mod 256, same tree.
 *   s_w    = 1 / max((float)(S / (N*K)), 1e-5)
 *   t      = clamp(rint(W * s_w), -1, 1)  stored as code t+1 in 2 bits;
 *            weight k of row n sits in bits [2(k%4), 2(k%4)+1] of byte
 *            W_packed[n*(K/4) + k/4].  Code 3 is never written.
 *   acc    = sum_k x_q[m,k] * t[n,k]   (int32, exact)
 *   y      = (float)acc / (s_x[m] * s_w)  (product rounded to fp32 first);
 *            bf16 output = round-to-nearest-even of that fp32 value.
 *
 * Layouts: row-major, x [M][K], W [N][K] (y = x W^T as in a linear layer),
 * W_packed [N][K/4] bytes, x_q [M][K] int8, acc and y [M][N].
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library allocates nothing and never synchronises (except the two
 *     status calls that say so).  Work is queued on `stream` (a
 *     cudaStream_t; NULL = the legacy default stream) and runs
 *     asynchronously.
 *   - Shapes: 0 <= M <= BITNET_MAX_M (M == 0 queues nothing and returns
 *     BITNET_OK), 1 <= N <= BITNET_MAX_N, 64 <= K <= BITNET_MAX_K and
 *     K % 64 == 0; outside these, BITNET_ERR_UNSUPPORTED_SHAPE.
 *   - Every tensor pointer must be 16-byte aligned (workspace: 256-byte).
 *   - Invalid arguments return a status and queue nothing.
 *   - Errors of the CUDA launch itself return BITNET_ERR_CUDA.
 *   - Kernels that wait on on-chip barriers give up after a bounded time,
 *     record BITNET_ERR_TIMEOUT in a device status word and exit cleanly;
 *     bitnet_device_status() reads it.
 */
#ifndef BITNET_B200_H
#define BITNET_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define BITNET_API __attribute__((visibility("default")))
#else
#define BITNET_API
#endif

/* cudaStream_t without pulling in the CUDA headers. */
typedef struct CUstream_st *bitnet_stream_t;

typedef enum {
    BITNET_OK = 0,
    BITNET_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad dtype, eps < 0 */
    BITNET_ERR_UNSUPPORTED_SHAPE = 2, /* K % 64 != 0, K, M or N out of range */
    BITNET_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte (workspace 256-byte) aligned */
    BITNET_ERR_CUDA = 4,              /* a CUDA launch or query failed */
    BITNET_ERR_TIMEOUT = 5,           /* a bounded on-device wait gave up */
    BITNET_ERR_WORKSPACE = 6,         /* workspace missing or too small */
    BITNET_ERR_SCRATCH_LIMIT = 7      /* N above BITNET_STATIC_SCRATCH_MAX_N (static-scratch call) */
} bitnet_status;

typedef enum { BITNET_F32 = 0, BITNET_BF16 = 1 } bitnet_dtype;

/* Matmul path selection for the debug entry point (results never depend on it). */
typedef enum {
    BITNET_PATH_AUTO = 0,  /* decode GEMV for M <= 16 and <= 32 MB of packed weights, else tcgen05 */
    BITNET_PATH_GEMV = 1,  /* streaming decode matmul (mma.sync; dp4a for M = 1 on tiled
                              weights); needs M <= 16 */
    BITNET_PATH_GEMM = 2   /* tcgen05 + TMA GEMM with TMEM accumulators */
} bitnet_path;

/* Layout of the packed weights a forward reads (see bitnet_tile_weights). */
typedef enum {
    BITNET_LAYOUT_ROWS = 0,   /* W_packed [N][K/4], the exported layout */
    BITNET_LAYOUT_TILED = 1   /* 128-row x 256-k tiles, bitnet_tile_weights */
} bitnet_layout;

#define BITNET_MAX_K (1 << 20)
/* Token rows of one call: 65535 tiles of 128 tokens (the tensor-core grid's
 * token dimension); weight rows: 2^24. */
#define BITNET_MAX_M (65535 * 128)
#define BITNET_MAX_N (1 << 24)

/* Human-readable name of a status code (static string, never NULL). */
BITNET_API const char *bitnet_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
BITNET_API int bitnet_version(void);

/* The CUDA runtime error code (cudaError_t) behind the last
 * BITNET_ERR_CUDA a call of this thread returned, 0 if none since the last
 * query; *name (may be NULL) receives the runtime's name for it.  Clears the
 * record. */
BITNET_API int bitnet_last_cuda_error(const char **name);

/* ------------------------------------------------------------------------
 * bitnet_quantize_pack_weights -- absmean ternary quantization + packing.
 * (first page, 量子化の仕組み weights bullet; The Era of 1-bit LLMs review,
 *  提案手法; packing: first page, 主な発見.)
 *
 *   W          [N][K] fp32 in.
 *   W_packed   [N][K/4] bytes out (layout above).
 *   s_w        one fp32 out (device memory): the per-tensor scale 1/mean|W|.
 *   workspace  >= bitnet_quantize_pack_weights_workspace_bytes(N, K) bytes of
 *              device scratch (fp64 row sums); contents on entry don't matter.
 * Deterministic: the same W gives the same bytes and s_w on every call.
 * ---------------------------------------------------------------------- */
BITNET_API size_t bitnet_quantize_pack_weights_workspace_bytes(int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_quantize_pack_weights(const float *W, int64_t N, int64_t K,
                                                      uint8_t *W_packed, float *s_w,
                                                      void *workspace, size_t workspace_bytes,
                                                      bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_quantize_pack_weights_static -- the same quantization and packing
 * as bitnet_quantize_pack_weights (identical bytes and s_w), but it needs no
 * workspace and allocates nothing.  The pages have no counterpart: this only
 * changes where the kernels' scratch lives.
 *
 * Why: some callers cannot call cudaMalloc -- plugins run by an inference
 * engine that owns the whole device-memory budget and hands its plugins only
 * their input and output tensors; code that must not risk the device-wide
 * synchronisation that cudaMalloc/cudaFree may cause; processes whose memory
 * is reserved up front by a capped pool.  Such callers still pass W,
 * W_packed and s_w (their own buffers).
 *
 * Scratch: a file-scope device array of BITNET_STATIC_SCRATCH_MAX_N fp64
 * row sums (512 KiB) inside the library, which every GPU that loads the
 * library holds until the process exits.  Limit: N <= 65536 rows; a larger N
 * returns BITNET_ERR_SCRATCH_LIMIT and queues nothing.  Every row sum is
 * written before it is read, so nothing in the array needs clearing between
 * calls, but all calls on a device share the one array: calls whose kernels
 * overlap on the GPU (different streams without ordering between them) race
 * and may produce wrong scales.  Order such calls on one stream.
 *
 * Set-up: the first call on each device looks up the array's device address
 * (with that device current) and keeps it for the process; make that first
 * call before any stream capture on the device.
 * Other arguments, layouts and errors as bitnet_quantize_pack_weights.
 * ---------------------------------------------------------------------- */
#define BITNET_STATIC_SCRATCH_MAX_N 65536
BITNET_API bitnet_status bitnet_quantize_pack_weights_static(const float *W, int64_t N,
                                                             int64_t K, uint8_t *W_packed,
                                                             float *s_w,
                                                             bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_tile_weights -- rearrange packed weights into the tiled layout the
 * matmul kernels stream fastest (an offline step, like the packing itself;
 * first page, 主な発見: the packed weights are stored for the kernels, and
 * 推論最適化とカスタムカーネル / タイル化行列乗算: the kernels read them
 * tile by tile).  The codes are unchanged; only their order is:
 *
 *   RB = ceil(N/128) row blocks, KC = ceil(K/256) k chunks; tile (rb, c)
 *   occupies bytes [(rb*KC + c) * 8192, +8192) of W_tiled.  Inside a tile,
 *   row r (0..127) is 64 bytes = four 16-byte pieces, piece q holding the
 *   packed bytes of weights k = 256c + 64q .. +63 of row 128*rb + r (i.e.
 *   W_packed[(128*rb + r)*K/4 + 64c + 16q .. +16]) at byte
 *   r*64 + 16*(q ^ ((r >> 1) & 3)).  Rows >= N and weights >= K are zero.
 *
 * With this layout a run of tiles of one row block is one contiguous range,
 * which a copy engine moves in one operation.
 *
 *   W_packed  [N][K/4] bytes in (device).
 *   W_tiled   bitnet_tiled_weights_bytes(N, K) bytes out (device, 16-byte
 *             aligned), caller-owned.
 * Shape rules as every entry point; returns 0 from the size query for an
 * unsupported shape.  Queues one kernel on `stream`.
 * ---------------------------------------------------------------------- */
BITNET_API size_t bitnet_tiled_weights_bytes(int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_tile_weights(const uint8_t *W_packed, int64_t N, int64_t K,
                                             uint8_t *W_tiled, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_tile_weights_pair -- the pair-tiled layout of two packed matrices
 * of the same shape [N][K/4] (the gate and up projections of a SwiGLU, The
 * Era of 1-bit LLMs review, 提案手法): unit (rb, c), at bytes
 * [(rb*KC + c) * 16384, +16384), is tile (rb, c) of Wa (layout of
 * bitnet_tile_weights) followed by tile (rb, c) of Wb.  Codes unchanged.
 *   W_pair  bitnet_tiled_pair_weights_bytes(N, K) bytes out (16-byte aligned).
 * ---------------------------------------------------------------------- */
BITNET_API size_t bitnet_tiled_pair_weights_bytes(int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_tile_weights_pair(const uint8_t *Wa_packed,
                                                  const uint8_t *Wb_packed, int64_t N, int64_t K,
                                                  uint8_t *W_pair, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_swiglu_forward -- the feed-forward's gate and up BitLinear forwards
 * of one input and the SwiGLU that joins them, y = silu(gate) * up with
 * silu(z) = z / (1 + e^-z) (The Era of 1-bit LLMs review, 提案手法: SwiGLU in
 * the LLaMA-like block; each forward as bitnet_linear_forward).  One
 * activation-quant launch and one matmul launch that computes both
 * projections of every output row and applies the activation in its
 * epilogue: gate and up are bit-identical to two separate forwards (fp32),
 * the activation is computed in fp32 (expf, then IEEE add, divide and
 * multiply; within a few fp32 ulp of the exact value).
 *
 *   W_pair                 pair-tiled gate/up weights (bitnet_tile_weights_pair).
 *   s_w_gate, s_w_up       their scales (device, one fp32 each).
 *   M                      0 <= M <= 16 (decode); larger M returns
 *                          BITNET_ERR_UNSUPPORTED_SHAPE.
 *   y                      [M][N] out, fp32 or bf16.
 *   workspace              >= bitnet_swiglu_forward_workspace_bytes(M, N, K),
 *                          256-byte aligned, contents on entry irrelevant.
 * ---------------------------------------------------------------------- */
BITNET_API size_t bitnet_swiglu_forward_workspace_bytes(int64_t M, int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_swiglu_forward(const void *x, int x_dtype, const float *gamma,
                                               float eps, const uint8_t *W_pair,
                                               const float *s_w_gate, const float *s_w_up,
                                               int64_t M, int64_t N, int64_t K, void *y,
                                               int y_dtype, void *workspace,
                                               size_t workspace_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_rmsnorm_quant_act -- fused RMSNorm + per-token absmax int8 quant.
 * (first page, 量子化の仕組み activations bullet; The Era of 1-bit LLMs
 *  review, 提案手法 RMSNorm; bitnet.cpp article, 数学的基礎 item 2.)
 *
 *   x        [M][K], fp32 or bf16 per x_dtype.
 *   gamma    [K] fp32 RMSNorm gain, or NULL for all ones.
 *   eps      >= 0, added to the mean square.
 *   x_q      [M][K] int8 out (natural k order).
 *   s_x      [M] fp32 out, 127 / max|x_n| per token.
 * ---------------------------------------------------------------------- */
BITNET_API bitnet_status bitnet_rmsnorm_quant_act(const void *x, int x_dtype, const float *gamma,
                                                  float eps, int64_t M, int64_t K, int8_t *x_q,
                                                  float *s_x, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_linear_forward -- the whole BitLinear forward, y = dequant(
 *   quant(rmsnorm(x)) * ternary(W)^T ).  Picks the warp-MMA decode GEMV for
 *   M <= 16 with at most 32 MB of packed weights and the tcgen05 kernel
 *   otherwise; both give identical bits.
 *   (The steps: first page, 量子化の仕組み -- normalise, absmax-quantize the
 *    activations, ternary weights, rescale by both scales; 計算パラダイム --
 *    integer additions in place of floating-point multiply-adds; 推論最適化と
 *    カスタムカーネル -- weights unpacked on the fly inside the matmul; The Era
 *    of 1-bit LLMs review, 提案手法 -- RMSNorm and absmean.)
 *
 *   x, x_dtype, gamma, eps   as bitnet_rmsnorm_quant_act.
 *   W_packed, s_w            as produced by bitnet_quantize_pack_weights
 *                            (s_w is read on the device).
 *   y                        [M][N] out, fp32 or bf16 per y_dtype.
 *   workspace                >= bitnet_linear_forward_workspace_bytes(M,N,K)
 *                            bytes, 256-byte aligned; its contents on entry
 *                            do not matter (the call clears what must start
 *                            at zero).  Calls that share a workspace must not
 *                            overlap in time (use one per stream).
 * ---------------------------------------------------------------------- */
BITNET_API size_t bitnet_linear_forward_workspace_bytes(int64_t M, int64_t N, int64_t K);
/* The same size under the short name the forward's plan gives it (identical
 * result for every M, N, K). */
BITNET_API size_t bitnet_workspace_bytes(int64_t M, int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_linear_forward(const void *x, int x_dtype, const float *gamma,
                                               float eps, const uint8_t *W_packed,
                                               const float *s_w, int64_t M, int64_t N, int64_t K,
                                               void *y, int y_dtype, void *workspace,
                                               size_t workspace_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * The forward in two phases, for callers that reuse one quantized input for
 * several weight matrices (e.g. the q, k and v projections of one token
 * batch) or time the phases separately.  bitnet_linear_forward(...) queues
 * exactly bitnet_linear_quantize_input(...) followed by
 * bitnet_linear_matmul(...).
 *
 * bitnet_linear_quantize_input -- RMSNorm + absmax int8 quant of x into the
 *   workspace (the kernels' internal layout: x_q k-interleaved inside
 *   16-element groups, s_x, per-token sums of x_q).  Arguments as
 *   bitnet_linear_forward; N is the largest output width the workspace will
 *   serve (it only sizes the workspace).
 * bitnet_linear_matmul -- integer matmul of the workspace's quantized input
 *   with W_packed and the fused dequant into y.  M and K must equal those of
 *   the preceding bitnet_linear_quantize_input on the same workspace, N must
 *   not exceed the N given to it, and workspace_bytes must cover (M, N, K).
 *   Any number of matmuls may follow one quantize call, in stream order.
 * ---------------------------------------------------------------------- */
BITNET_API bitnet_status bitnet_linear_quantize_input(const void *x, int x_dtype,
                                                      const float *gamma, float eps, int64_t M,
                                                      int64_t N, int64_t K, void *workspace,
                                                      size_t workspace_bytes,
                                                      bitnet_stream_t stream);
BITNET_API bitnet_status bitnet_linear_matmul(const uint8_t *W_packed, const float *s_w,
                                              int64_t M, int64_t N, int64_t K, void *y,
                                              int y_dtype, void *workspace,
                                              size_t workspace_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_linear_forward_grouped -- several independent BitLinear forwards in
 * one call (each one the forward of the first page's 量子化の仕組み, as
 * bitnet_linear_forward; the projections of one LLaMA-like block, The Era of
 * 1-bit LLMs review, 提案手法, are the typical group): the result is exactly
 * that of calling bitnet_linear_forward on each problem in order, but every
 * problem's activation quantization is one launch and the decode problems
 * (M <= 16) share one matmul launch, so their weight streams overlap instead
 * of paying one launch latency each.  Typical use: the projections of one
 * decode step (q, k, v, o, gate, up, down).  Problems with the same x,
 * x_dtype, gamma, eps, M and K (q/k/v, gate/up) that use the same matmul
 * kind share one activation quantization.  The host-side plan of a call is
 * cached per thread (a few entries, keyed by every field of every problem
 * and the workspace), so a decode loop that repeats the same call plans it
 * once.  The matmuls of problems with M > 16 run afterwards on the tcgen05
 * kernel, one at a time.
 *
 *   count      0 <= count <= BITNET_MAX_GROUP.
 *   problems   host array of `count` problem descriptions (each field as in
 *              bitnet_linear_forward).  No problem's y may overlap another
 *              problem's inputs or output.
 *   workspace  >= bitnet_linear_forward_grouped_workspace_bytes(count,
 *              problems), 256-byte aligned, contents on entry irrelevant.
 *   phases     BITNET_PHASE_ALL, or one phase at a time: BITNET_PHASE_QUANTIZE
 *              (activation quant of every problem into the workspace) then,
 *              later on the same stream with the same problems and
 *              workspace, BITNET_PHASE_MATMUL (every matmul).  Splitting
 *              lets a caller time the phases or reuse one quantization; the
 *              results are identical.
 * Any invalid problem rejects the whole call before anything is queued.
 * ---------------------------------------------------------------------- */
#define BITNET_MAX_GROUP 16
#define BITNET_PHASE_QUANTIZE 1
#define BITNET_PHASE_MATMUL 2
#define BITNET_PHASE_ALL 3
typedef struct {
    const void *x;            /* [M][K] */
    int x_dtype;              /* bitnet_dtype */
    const float *gamma;       /* [K] or NULL */
    float eps;
    const uint8_t *W_packed;  /* [N][K/4] row-major, or the tiled layout (w_layout) */
    const float *s_w;         /* [1] */
    int64_t M, N, K;
    void *y;                  /* [M][N] */
    int y_dtype;              /* bitnet_dtype */
    int w_layout;             /* bitnet_layout of W_packed (zero = row-major) */
} bitnet_linear_problem;

BITNET_API size_t bitnet_linear_forward_grouped_workspace_bytes(
    int count, const bitnet_linear_problem *problems);
BITNET_API bitnet_status bitnet_linear_forward_grouped(int count,
                                                       const bitnet_linear_problem *problems,
                                                       void *workspace, size_t workspace_bytes,
                                                       int phases, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_linear_forward_debug -- bitnet_linear_forward that also exports the
 * intermediate results, and can force a matmul path.  (The exported values
 * are the quantized activations of the first page's 量子化の仕組み
 * activations bullet and the integer accumulators of its 計算パラダイム.)
 *
 *   x_q_out  [M][K] int8 (natural k order) or NULL.
 *   s_x_out  [M] fp32 or NULL.
 *   acc_out  [M][N] int32 accumulators (before dequant) or NULL.
 *   y        may be NULL (then only the debug outputs are written).
 *   path     a bitnet_path value.
 * ---------------------------------------------------------------------- */
BITNET_API bitnet_status bitnet_linear_forward_debug(
    const void *x, int x_dtype, const float *gamma, float eps, const uint8_t *W_packed,
    const float *s_w, int64_t M, int64_t N, int64_t K, void *y, int y_dtype, void *workspace,
    size_t workspace_bytes, int8_t *x_q_out, float *s_x_out, int32_t *acc_out, int path,
    bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * Group-wise scales (bitnet.cpp article, グループ量子化と正規化: the weights
 * and the activations are split into groups quantized independently, so
 * that the groups need no communication).  Reading: G = K / group_k
 * contiguous groups along K, group_k a multiple of 256 with G <= 512:
 *   s_w[g]   = 1 / max(mean |W| over all rows and the group's columns, 1e-5)
 *              (fp64 sum in the order of the per-tensor scale, applied to the
 *              N x group_k block of group g)
 *   t        = clamp(rint(W * s_w[g(k)]), -1, 1), packed as W_packed
 *   x_n      = RMSNorm of the whole row (as bitnet_rmsnorm_quant_act)
 *   s_x[m,g] = 127 / max(max over the group of |x_n|, 1e-5)
 *   x_q      = clamp(rint(x_n * s_x[m,g(k)]), -128, 127)
 *   acc_g    = sum over the group of x_q * t            (int32, exact)
 *   y[m,n]   = sum_g (float)acc_g / (s_x[m,g] * s_w[g]): fp32 terms (product
 *              rounded first, correctly rounded division) summed in fp64 in
 *              increasing g and rounded once to fp32.
 * With group_k = K this is the per-tensor forward bit for bit.
 *
 * bitnet_quantize_pack_weights_group_scales -- W [N][K] fp32 -> W_packed
 *   [N][K/4], s_w [G] (device); workspace >= the size query (fp64 row sums).
 * bitnet_linear_forward_group_scales -- the forward.  W_packed in either
 *   layout (w_layout, a bitnet_layout); the tiled decode kernel serves tiled
 *   weights with M <= 16, the tcgen05 kernel the rest, one K split per group;
 *   both write the groups' integer sums and a last kernel forms y.
 *   y          [M][N] fp32 or bf16, or NULL when acc_out is given.
 *   x_q_out    [M][K] int8 natural order, s_x_out [M][G] fp32, acc_out
 *              [G][M][N] int32 (the group sums): optional debug exports.
 *   workspace  >= bitnet_linear_forward_group_scales_workspace_bytes, 256-byte
 *              aligned, contents on entry irrelevant.
 * Unsupported group_k -> BITNET_ERR_UNSUPPORTED_SHAPE.
 * ---------------------------------------------------------------------- */
BITNET_API size_t bitnet_quantize_pack_weights_group_scales_workspace_bytes(int64_t N,
                                                                            int64_t K,
                                                                            int64_t group_k);
BITNET_API bitnet_status bitnet_quantize_pack_weights_group_scales(
    const float *W, int64_t N, int64_t K, int64_t group_k, uint8_t *W_packed, float *s_w,
    void *workspace, size_t workspace_bytes, bitnet_stream_t stream);
BITNET_API size_t bitnet_linear_forward_group_scales_workspace_bytes(int64_t M, int64_t N,
                                                                     int64_t K,
                                                                     int64_t group_k);
BITNET_API bitnet_status bitnet_linear_forward_group_scales(
    const void *x, int x_dtype, const float *gamma, float eps, const uint8_t *W_packed,
    int w_layout, const float *s_w, int64_t M, int64_t N, int64_t K, int64_t group_k, void *y,
    int y_dtype, void *workspace, size_t workspace_bytes, int8_t *x_q_out, float *s_x_out,
    int32_t *acc_out, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * Quantization warm-up for fine-tuning ("LLM を 1.58 ビットにファインチューニ
 * ング：BitNet による極端な量子化", section 動的ウォームアップ量子化: lambda =
 * min(step / total_steps, 1) scales the difference between the full-precision
 * and the quantized values; the straight-through estimator of the same page
 * for the backward).  Reading: the blend applies to both operands the page
 * quantizes, in rounded fp32 steps, each rounded to bf16 for the tensor cores:
 *   W_lam = W + lambda * (t / s_w - W)         t, s_w as bitnet_quantize_pack_weights
 *   x_lam = x_n + lambda * (x_q / s_x - x_n)   x_n, x_q, s_x as bitnet_rmsnorm_quant_act
 *   y     = x_lam W_lam^T                       bf16 operands, fp32 accumulation
 * lambda = 0 is the plain bf16 layer on the normalised input; lambda = 1 is
 * the fake-quantized layer (y = the dequantized ternary forward up to the
 * bf16 rounding of x_q / s_x and t / s_w and fp32 summation order).
 * Shapes: N and K multiples of 8, 0 <= lambda <= 1.
 *
 * bitnet_warmup_quantize_weights -- W [N][K] fp32 (device, 16-byte aligned)
 *   -> W_lam [N][K] bf16 and s_w [1] fp32; workspace >= the size query.
 * bitnet_warmup_forward -- x [M][K] (fp32 or bf16), gamma [K] or NULL,
 *   W_lam from the call above -> y [M][N] (y_dtype).  x_lam [M][K] bf16 is
 *   written to x_lam when it is non-NULL (kept for the backward), else to the
 *   workspace (>= bitnet_warmup_forward_workspace_bytes, 256-byte aligned).
 * bitnet_warmup_backward -- the straight-through backward of y = x_lam
 *   W_lam^T given dy [M][N] bf16: dx [M][K] fp32 = dy W_lam (the gradient
 *   of x_n; the RMSNorm's own backward is not part of this layer) and dW
 *   [N][K] fp32 = dy^T x_lam (the gradient of W, the quantizer passing it
 *   through).  Either output may be NULL.  workspace >= the size query
 *   (transposed bf16 copies).
 * All calls queue work on `stream` and return at once; device buffers only.
 * ---------------------------------------------------------------------- */
BITNET_API size_t bitnet_warmup_quantize_weights_workspace_bytes(int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_warmup_quantize_weights(const float *W, int64_t N, int64_t K,
                                                        float lambda, void *W_lam, float *s_w,
                                                        void *workspace, size_t workspace_bytes,
                                                        bitnet_stream_t stream);
BITNET_API size_t bitnet_warmup_forward_workspace_bytes(int64_t M, int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_warmup_forward(const void *x, int x_dtype, const float *gamma,
                                               float eps, const void *W_lam, int64_t M,
                                               int64_t N, int64_t K, float lambda, void *y,
                                               int y_dtype, void *x_lam, void *workspace,
                                               size_t workspace_bytes, bitnet_stream_t stream);
BITNET_API size_t bitnet_warmup_backward_workspace_bytes(int64_t M, int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_warmup_backward(const void *dy, const void *x_lam,
                                                const void *W_lam, int64_t M, int64_t N,
                                                int64_t K, float *dx, float *dW, void *workspace,
                                                size_t workspace_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * BitDelta ("【論文要約】BitDelta: Your Fine-Tune May Only Be Worth One Bit",
 * Eq. 1-4: Delta = W_fine - W_base is stored as its sign and one scale per
 * matrix, alpha = mean |Delta|; Eq. 6 and Fig. 4: a shared base matrix
 * serves B tenants at once, each token through base + its tenant's delta).
 * Readings: Sign(0) = -1; bit j (least significant first) of word w of row n
 * is the sign of Delta[n][32 w + j] (1 = +1); alpha is the fp64 sum of |Delta|
 * in the fixed order of the weight scale divided by N K, rounded to fp32.
 *
 * bitnet_bitdelta_compress -- W_base, W_fine [N][K] bf16 (device, 16-byte
 *   aligned), K a multiple of 32 -> signs [N][K/32] uint32 and alpha [1]
 *   fp32; workspace >= the size query (fp64 row sums).
 * bitnet_bitdelta_forward -- B <= 8 tenants, one token each: x [B][K] bf16,
 *   W_base [N][K] bf16, signs [B][N][K/32] (tenant after tenant), alpha [B]
 *   -> y [B][N] (y_dtype) with
 *     y[b][n] = sum_k x[b][k] W_base[n][k] + alpha[b] sum_k x[b][k] s_b[n][k]
 *   (bf16 products, fp32 sums on the tensor cores, the delta's sum scaled
 *   by alpha with one fused multiply-add).  B == 0 queues nothing.
 * ---------------------------------------------------------------------- */
BITNET_API size_t bitnet_bitdelta_compress_workspace_bytes(int64_t N, int64_t K);
BITNET_API bitnet_status bitnet_bitdelta_compress(const void *W_base, const void *W_fine,
                                                  int64_t N, int64_t K, uint32_t *signs,
                                                  float *alpha, void *workspace,
                                                  size_t workspace_bytes,
                                                  bitnet_stream_t stream);
BITNET_API bitnet_status bitnet_bitdelta_forward(const void *x, const void *W_base,
                                                 const uint32_t *signs, const float *alpha,
                                                 int64_t B, int64_t N, int64_t K, void *y,
                                                 int y_dtype, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_linear_forward_ex -- one forward described by a problem record, so
 * that it can read weights in either layout (problem->w_layout); otherwise
 * as bitnet_linear_forward_debug: the same steps, the same bits, optional
 * exports of x_q (natural order), s_x and the int32 accumulators, and a
 * matmul path selector.  problem->y may be NULL when acc_out is given.
 * With tiled weights the automatic path takes the tiled decode kernel for
 * every M <= 16 and the tcgen05 kernel above.
 *
 *   workspace  >= bitnet_linear_forward_workspace_bytes(M, N, K).
 * ---------------------------------------------------------------------- */
BITNET_API bitnet_status bitnet_linear_forward_ex(const bitnet_linear_problem *problem,
                                                  void *workspace, size_t workspace_bytes,
                                                  int8_t *x_q_out, float *s_x_out,
                                                  int32_t *acc_out, int path,
                                                  bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_ternary_matmul_i32 -- debug: acc = x_q * t^T on the integer path
 * alone (first page, 計算パラダイム).  Unlike a plain (x_q, W_packed, acc)
 * signature it takes a workspace (the library allocates nothing; the
 * kernels need the activations in their interleaved order and, for few
 * rows, split-K partials) and a path selector (to check both kernels).
 *
 *   x_q       [M][K] int8 (natural k order, any values in [-128, 127]).
 *   W_packed  [N][K/4].
 *   acc       [M][N] int32 out.
 *   workspace >= bitnet_linear_forward_workspace_bytes(M,N,K) (same contract
 *             as the forward).
 *   path      a bitnet_path value.
 * ---------------------------------------------------------------------- */
BITNET_API bitnet_status bitnet_ternary_matmul_i32(const int8_t *x_q, const uint8_t *W_packed,
                                                   int64_t M, int64_t N, int64_t K, int32_t *acc,
                                                   void *workspace, size_t workspace_bytes,
                                                   int path, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * Device status word.  bitnet_device_status synchronises `stream`, returns
 * BITNET_OK or the first BITNET_ERR_TIMEOUT recorded by a kernel since the
 * last reset, stores the kernel-side detail code in *detail (may be NULL),
 * and clears the word when reset != 0.  It is per device and per process.
 * ---------------------------------------------------------------------- */
BITNET_API bitnet_status bitnet_device_status(bitnet_stream_t stream, int reset, int *detail);
/* bitnet_device_status(stream, 0, NULL): synchronises `stream` and returns
 * the recorded status without clearing it. */
BITNET_API bitnet_status bitnet_last_device_status(bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_selftest_bounded_wait -- runs one tiny kernel that waits on an
 * on-chip barrier nothing ever completes, with the given limit in
 * nanoseconds (1e3..1e9), so callers can check that bounded waits end and
 * report BITNET_ERR_TIMEOUT through bitnet_device_status.  It does not touch
 * any tensor.  Queues on `stream`.
 * ---------------------------------------------------------------------- */
BITNET_API bitnet_status bitnet_selftest_bounded_wait(uint64_t limit_ns, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_selftest_divide -- q[i] = a[i] / b[i] through the division the
 * dequant epilogues use for y = acc / (s_x * s_w): the correctly rounded
 * reciprocal of b and two fused residual corrections (Markstein's method),
 * which rounds to nearest even exactly like an IEEE binary32 division when
 * 2^-95 <= |b| <= 2^100 and a is 0 or 1 <= |a| <= 2^31 (every numerator the
 * dequant produces is an integer in that range, so the epilogues check only
 * the divisor, once per token); any other pair takes the IEEE division.
 * Lets a test check that the result always equals a host IEEE division.
 *
 *   a, b, q   device fp32 arrays of n elements (16-byte aligned), caller-owned.
 *   n         >= 0.
 * Queues one kernel on `stream`; BITNET_ERR_INVALID_ARG / _MISALIGNED on bad
 * arguments (nothing queued).
 * ---------------------------------------------------------------------- */
BITNET_API bitnet_status bitnet_selftest_divide(const float *a, const float *b, float *q,
                                                int64_t n, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_selftest_mma_i8 -- measurement aid, not part of the forward: queues
 * one kernel of `ctas` CTAs (one per SM for a whole-GPU figure), each
 * issuing `iters` back-to-back int8 tensor-core MMAs of shape 128 x 256 x 32
 * (tcgen05.mma kind::i8, A from shared memory, or from tensor memory like
 * the forward's kernels when a_in_tmem != 0) on zero data.  Timing it with
 * events on `stream` gives the dense int8 rate of the GPU as clocked:
 * int8 operations = 2 * 128 * 256 * 32 * iters * ctas.  Touches no tensor.
 *   iters  1 .. 1e8;  ctas  1 .. 65535.
 * ---------------------------------------------------------------------- */
BITNET_API bitnet_status bitnet_selftest_mma_i8(int64_t iters, int ctas, int a_in_tmem,
                                                bitnet_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_B200_H */
