// tile.cuh -- 64 x 128 bf16 tiles streamed through shared memory with
// cp.async, shared by the tile kernels of the NVFP4 and MXFP4 quantizers.
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

#include "nvfp4_device.cuh"

namespace nvfp4 {

// Tiles of 64 x 128 bf16 staged in shared memory, two buffers so the next
// tile streams in while this one is processed.  Chunk c (16 bytes) of tile
// row r is stored at slot (c ^ ((c >> 3) & 1)) ^ (2 ((r >> 4) & 3)): the
// eight lanes reading one row's eight 32-byte blocks hit 32 distinct banks,
// and so do 32 lanes reading one 32-bit column word each from 8 columns
// pairs x 4 row blocks, or from 32 column pairs of one row.
constexpr int TR = 64, TC = 128, TNT = 256;

__device__ __forceinline__ int tile_chunk(int r, int c) { return (c ^ ((c >> 3) & 1)) ^ (((r >> 4) & 3) << 1); }
// 32-bit word w (columns 2w, 2w + 1) of tile row r
__device__ __forceinline__ int tile_word(int r, int w) { return (tile_chunk(r, w >> 2) << 2) | (w & 3); }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// Tile index -> (tile row, tile column) of the row-major tile grid.
__device__ __forceinline__ void tile_coords(uint32_t tile, const FastDiv& tiles_c, int64_t& tr, int64_t& tc) {
  const uint32_t q = fastdiv(tile, tiles_c);
  tr = q;
  tc = tile - q * tiles_c.d;
}

// 2D-block layout: chunk c of row r at slot c ^ (r & 7), so that the eight
// lanes reading one chunk column of eight consecutive rows hit 32 distinct
// banks, as do 32 lanes reading 32 consecutive words of one row.
__device__ __forceinline__ int tile_chunk_2d(int r, int c) { return c ^ (r & 7); }
__device__ __forceinline__ int tile_word_2d(int r, int w) { return (tile_chunk_2d(r, w >> 2) << 2) | (w & 3); }

// Issue the copies of tile `tile` (row-major tile grid) into buf, in the
// 1D (SW2D = false) or the 2D-block (SW2D = true) layout, by NT threads.
// Thread t copies chunk cc = t % 16 of rows t / 16 + (NT / 16) i
// (i < 16 TR / NT): one 64-bit address for the first row, the others NT / 16
// rows apart.
template <bool SW2D = false, int NT = TNT>
__device__ __forceinline__ void load_tile_at(uint4 (*buf)[TC / 8], const uint16_t* x, int64_t R, int64_t C,
                                             int64_t ld, uint32_t tr, uint32_t tc) {
  constexpr int kRowStep = NT / 16, kPasses = TR / kRowStep;
  const int64_t r0 = static_cast<int64_t>(tr) * TR, c0 = static_cast<int64_t>(tc) * TC;
  const int row0 = static_cast<int>(threadIdx.x) >> 4, cc = static_cast<int>(threadIdx.x) & 15;
  const uint16_t* src = x + (r0 + row0) * ld + c0 + 8 * cc;
  const int64_t step = kRowStep * ld;
  if (R - r0 >= TR && C - c0 >= TC) {
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
      const int row = row0 + kRowStep * i;
      cp_async16(&buf[row][SW2D ? tile_chunk_2d(row, cc) : tile_chunk(row, cc)], src + i * step);
    }
  } else {
    const int rows = static_cast<int>(R - r0 < TR ? R - r0 : TR);
    const int cols = static_cast<int>(C - c0 < TC ? C - c0 : TC);
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
      const int row = row0 + kRowStep * i;
      if (row < rows && 8 * cc < cols)
        cp_async16(&buf[row][SW2D ? tile_chunk_2d(row, cc) : tile_chunk(row, cc)], src + i * step);
    }
  }
  cp_async_commit();
}

template <bool SW2D = false>
__device__ __forceinline__ void load_tile_async(uint4 (*buf)[TC / 8], const uint16_t* x, int64_t R, int64_t C,
                                                int64_t ld, const FastDiv& tiles_c, uint32_t tile) {
  int64_t tr, tc;
  tile_coords(tile, tiles_c, tr, tc);
  load_tile_at<SW2D>(buf, x, R, C, ld, static_cast<uint32_t>(tr), static_cast<uint32_t>(tc));
}

// Coordinates of the tiles a CTA visits (tile, tile + step, ...) in the
// row-major grid of `tiles_c` tile columns, advanced without a division.
struct TileWalk {
  uint32_t tr, tc, dtr, dtc, tiles_c;
  __device__ __forceinline__ TileWalk(uint32_t tile, uint32_t step, uint32_t cols)
      : tr(tile / cols), tc(tile - (tile / cols) * cols), dtr(step / cols), dtc(step - (step / cols) * cols),
        tiles_c(cols) {}
  __device__ __forceinline__ void advance() {
    tc += dtc;
    tr += dtr;
    if (tc >= tiles_c) {
      tc -= tiles_c;
      ++tr;
    }
  }
};

}  // namespace nvfp4
