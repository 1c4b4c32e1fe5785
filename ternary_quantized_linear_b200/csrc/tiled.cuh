// tiled.cuh -- the tiled layout of packed ternary weights, and the kernel
// that produces it from the row-major packed bytes.
//
// The row-major layout W_packed [N][K/4] (weight k of row n in bits
// [2(k%4), 2(k%4)+1] of byte n*K/4 + k/4) is the exported format.  The
// matmul kernels read a weight matrix as tiles of 128 rows x 256 k (8 KiB
// of codes); in row-major order such a tile is 128 separate 64-byte pieces,
// so a copy engine needs one 2-D tensor copy per tile at best.  In the tiled
// layout every tile is contiguous and the tiles of a row block follow one
// another, so a whole run of tiles moves with one 1-D bulk copy, and the
// bytes of a tile are already in the shared-memory order the kernels read:
//
//   RB = ceil(N / 128) row blocks, KC = ceil(K / 256) k chunks;
//   tile (rb, c) starts at byte (rb * KC + c) * 8192;
//   inside it, row r (0..127) holds 64 bytes = four 16-byte pieces, and
//   piece q (weights k = 256 c + 64 q .. +63 of row 128 rb + r) sits at
//   byte r * 64 + 16 * (q ^ ((r >> 1) & 3)).
//   Rows past N and weights past K are zero bytes.
//
// The XOR spreads the pieces that the lanes of a warp read together over
// all 32 shared-memory banks (it is the 64-byte swizzle of the copy
// engine, applied once when the layout is built instead of on every copy).
// The tiling only moves bytes: the codes themselves are unchanged.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr int kTileRows = 128;
constexpr int kTileK = 256;
constexpr int kTileBytes = kTileRows * kTileK / 4;  // 8 KiB

__host__ __device__ constexpr int64_t tiled_row_blocks(int64_t N) { return (N + 127) / 128; }
__host__ __device__ constexpr int64_t tiled_chunks(int64_t K) { return (K + 255) / 256; }

// Byte offset, inside a 128-row x 256-k tile, of piece q of row r.
__host__ __device__ __forceinline__ int tile_piece_offset(int r, int q) {
  return r * 64 + 16 * (q ^ ((r >> 1) & 3));
}

// One thread per 16-byte piece of the tiled output (coalesced writes).
__global__ void __launch_bounds__(256)
tile_weights_kernel(const uint8_t* __restrict__ W_packed, int64_t N, int64_t K,
                    uint8_t* __restrict__ W_tiled, int64_t npieces) {
  const int64_t KC = tiled_chunks(K);
  const int64_t row_bytes = K / 4;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < npieces;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t tile = i >> 9;             // 512 pieces per tile
    const int j = static_cast<int>(i & 511);
    const int r = j >> 2, qp = j & 3;        // physical piece qp of row r
    const int q = qp ^ ((r >> 1) & 3);       // logical piece
    const int64_t rb = tile / KC, c = tile - rb * KC;
    const int64_t n = rb * kTileRows + r;
    const int64_t col = c * 64 + 16 * q;     // byte within the packed row
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (n < N && col < row_bytes)
      v = __ldg(reinterpret_cast<const uint4*>(W_packed + n * row_bytes + col));
    reinterpret_cast<uint4*>(W_tiled)[i] = v;
  }
}

// The pair-tiled layout of two matrices of the same shape (the gate and up
// projections of a SwiGLU): unit (rb, c) = tile (rb, c) of the first matrix
// followed by tile (rb, c) of the second, 16 KiB, units ordered as tiles.
__global__ void __launch_bounds__(256)
tile_pair_weights_kernel(const uint8_t* __restrict__ Wa, const uint8_t* __restrict__ Wb,
                         int64_t N, int64_t K, uint8_t* __restrict__ W_pair, int64_t npieces) {
  const int64_t KC = tiled_chunks(K);
  const int64_t row_bytes = K / 4;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < 2 * npieces;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t unit = i >> 10;            // 1024 pieces per unit
    const int which = static_cast<int>((i >> 9) & 1);
    const int j = static_cast<int>(i & 511);
    const int r = j >> 2, qp = j & 3;
    const int q = qp ^ ((r >> 1) & 3);
    const int64_t rb = unit / KC, c = unit - rb * KC;
    const int64_t n = rb * kTileRows + r;
    const int64_t col = c * 64 + 16 * q;
    const uint8_t* W = which ? Wb : Wa;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (n < N && col < row_bytes)
      v = __ldg(reinterpret_cast<const uint4*>(W + n * row_bytes + col));
    reinterpret_cast<uint4*>(W_pair)[i] = v;
  }
}

}  // namespace bitnet
