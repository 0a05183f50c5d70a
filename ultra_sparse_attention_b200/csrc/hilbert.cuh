// hilbert.cuh -- Hilbert-curve token order and the token permutation kernel.
//
// HilbertA blog page, "Introducing HilbertA", first component (Reordering):
// image tokens are put in the order of a Hilbert curve over the patch grid, so
// tokens that are close on the grid stay close in the sequence.  For the block
// mask that means a 64-token block of an image is an 8 x 8 patch square
// instead of a 64 x 1 strip of one patch row, which makes block pooling and
// the kept-block choice spatially coherent.  The attention path runs
// unchanged on the reordered tokens; the output is mapped back with the
// inverse permutation.
//
//   hilbert_index        host: a cell's position on the Hilbert curve of a
//                        2^k x 2^k square (top quadrant first, each level's
//                        remaining coordinates moved into the sub-square's
//                        own frame).
//   permute_rows_kernel  device: dst[bh][t] = src[bh][perm[t]] (gather) or
//                        dst[bh][perm[t]] = src[bh][t] (scatter), 16 bytes
//                        per thread; HBM-bound.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace rt {

// Position of cell (x, y) (x the column, y the row; both < 2^k) on the order-k curve that
// starts at (0, 0) and ends at (2^k - 1, 0).  The curve of side 2s visits the lower-left
// quadrant along its own transpose, then the upper-left and upper-right quadrants as is,
// then the lower-right quadrant along its anti-transpose; at each level the quadrant adds
// its quarter to the position and the coordinates are taken into that quadrant's frame.
inline uint64_t hilbert_index(int k, uint32_t x, uint32_t y) {
  uint64_t pos = 0;
  for (int level = k - 1; level >= 0; --level) {
    const uint32_t s = 1u << level;
    const bool right = x >= s, up = y >= s;
    const uint64_t quarter = static_cast<uint64_t>(s) * s;
    if (!right && !up) {  // lower left: transposed sub-curve
      const uint32_t t = x;
      x = y;
      y = t;
    } else if (!right && up) {  // upper left
      pos += quarter;
      y -= s;
    } else if (right && up) {  // upper right
      pos += 2 * quarter;
      x -= s;
      y -= s;
    } else {  // lower right: anti-transposed sub-curve
      pos += 3 * quarter;
      const uint32_t nx = s - 1 - y, ny = 2 * s - 1 - x;
      x = nx;
      y = ny;
    }
  }
  return pos;
}

// grid (ceil(N * D / 8 / 256), B*H), 256 threads; one 16-byte chunk per thread.  Entries of
// perm outside [0, N) are skipped (gather: the row is written as zeros).
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ perm,
                                                           uint4* __restrict__ dst, int N, int chunks_per_row,
                                                           int inverse) {
  if (device_status_set()) return;  // an earlier kernel failed
  const size_t per_head = static_cast<size_t>(N) * chunks_per_row;
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= per_head) return;
  const int t = static_cast<int>(idx / chunks_per_row), c = static_cast<int>(idx % chunks_per_row);
  const int p = __ldg(perm + t);
  const size_t head = static_cast<size_t>(blockIdx.y) * per_head;
  const bool in = p >= 0 && p < N;
  if (!inverse) {
    dst[head + idx] = in ? __ldg(src + head + static_cast<size_t>(p) * chunks_per_row + c) : make_uint4(0u, 0u, 0u, 0u);
  } else if (in) {
    dst[head + static_cast<size_t>(p) * chunks_per_row + c] = __ldg(src + head + idx);
  }
}

}  // namespace rt
