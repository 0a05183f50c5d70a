// pairing.cuh -- which two query blocks share a 128-row tile of the sparse step.
//
// The sparse kernel computes a 128-row query tile against the union of its
// query blocks' kept key blocks (block size 64: two query blocks per tile);
// a key block kept by only one of them costs the other half of the tile a
// wasted MMA and a key-tile step.  With the neighbouring pair (2t, 2t+1) on
// video-shaped inputs the two kept sets barely overlap apart from the forced
// prefix (13.9 key blocks per tile against 9 per query block at 9/278).
// This kernel pairs query blocks that keep many of the same key blocks
// instead (11.0 on the same inputs).  The pairing changes only which rows
// share a tile: every row's result is the same.
//
// Every step is deterministic:
//  1. candidates (pair_candidates_kernel, one CTA per kCandBlocks query blocks
//     of a head): for each query block i, the kPairCands best partners j with
//     |i - j| <= kPairWindow in the order (overlap desc, |i - j| asc, j asc),
//     where overlap = the number of key blocks both keep.  The kept sets of
//     the CTA's blocks and their window are bitmaps in shared memory, so an
//     overlap costs ceil(n_blocks / 32) AND + popcount steps whatever the
//     keep ratio; eight threads share a block's window and merge their lists;
//  2. mutual choice (pair_match_kernel, one CTA per head), kPairRounds
//     rounds: every unpaired block picks its first still-unpaired candidate;
//     two blocks that pick each other are paired;
//  3. tiles: the pairs in order of their lower block, then the blocks left
//     unpaired, two per tile in ascending order (the last one alone if their
//     count is odd; -1 marks the empty half).
// Block size 128 has one query block per tile: tile t is (t, -1).
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace rt {

constexpr int kPairCands = 8;
constexpr int kPairRounds = 8;
constexpr int kPairWindow = 224;
constexpr int kPairThreads = 256;
constexpr int kCandSplit = 8;                            // threads per query block in step 1
constexpr int kCandBlocks = kPairThreads / kCandSplit;  // query blocks per CTA in step 1

// Words of one kept-set bitmap row in shared memory: odd, so that rows a warp reads
// together fall in different banks.
__host__ __device__ constexpr int pairing_row_words(int n_blocks) { return ((n_blocks + 31) / 32) | 1; }

// Dynamic shared memory of pair_candidates_kernel: the bitmaps of a CTA's blocks and
// their window (133 KB at the 2048-block limit).
__host__ __device__ constexpr size_t pair_candidates_smem_bytes(int n_blocks) {
  return static_cast<size_t>(n_blocks < kCandBlocks + 2 * kPairWindow ? n_blocks : kCandBlocks + 2 * kPairWindow) *
         pairing_row_words(n_blocks) * 4;
}

// Dynamic shared memory of pair_match_kernel: candidates [n_blocks][kPairCands],
// partner and choice [n_blocks], all int16.
__host__ __device__ constexpr size_t pair_match_smem_bytes(int n_blocks) {
  return static_cast<size_t>(n_blocks) * (kPairCands + 2) * 2;
}

// Candidate order (overlap desc, |i - j| asc, j asc) as one integer, larger = better:
// key = overlap << 12 | (4095 - (2 |i - j| + [j > i])).  Keys of different partners
// differ, 0 is below every real key (2 |i - j| + 1 <= 2 kPairWindow + 1 < 4096 and an
// overlap is at most 2048).
__device__ __forceinline__ uint32_t pair_key(int ov, int dd, int side) {
  return (static_cast<uint32_t>(ov) << 12) | static_cast<uint32_t>(4095 - (2 * dd + side));
}

// Partner of block i encoded in `key` (-1 for the empty key 0).
__device__ __forceinline__ int pair_key_block(uint32_t key, int i) {
  if (key == 0u) return -1;
  const int code = 4095 - static_cast<int>(key & 4095u);
  return (code & 1) ? i + (code >> 1) : i - (code >> 1);
}

// Insert `x` into the descending list `k` (the smallest falls off): branch-free.
__device__ __forceinline__ void pair_insert(uint32_t (&k)[kPairCands], uint32_t x) {
#pragma unroll
  for (int c = 0; c < kPairCands; ++c) {
    const uint32_t hi = max(k[c], x);
    x = min(k[c], x);
    k[c] = hi;
  }
}

// Step 1.  grid (ceil(n_blocks / kCandBlocks), B*H), kPairThreads threads,
// pair_candidates_smem_bytes(n_blocks) dynamic shared memory; kMaxWords >= ceil(n_blocks / 32)
// (block i's bitmap is held in registers).
// cand: int16 [B*H][n_blocks][kPairCands], -1 = none.
template <int kMaxWords>
__global__ void __launch_bounds__(kPairThreads)
    pair_candidates_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx, int n_blocks,
                           int16_t* __restrict__ cand) {
  extern __shared__ uint32_t pair_bits[];  // [window rows][row_words]
  __shared__ int skip;
  if (threadIdx.x == 0) skip = device_status_set() ? 1 : 0;
  __syncthreads();
  if (skip) return;  // an earlier kernel failed (block-uniform)
  const int nb = n_blocks, bh = blockIdx.y, tid = threadIdx.x;
  const int words = (nb + 31) / 32, row_words = pairing_row_words(nb);
  const size_t row0 = static_cast<size_t>(bh) * nb;
  const int c0 = blockIdx.x * kCandBlocks;
  const int base = max(0, c0 - kPairWindow), top = min(nb, c0 + kCandBlocks + kPairWindow);
  for (int b = base + tid; b < top; b += kPairThreads) {
    uint32_t* row = pair_bits + static_cast<size_t>(b - base) * row_words;
    for (int w = 0; w < words; ++w) row[w] = 0u;
    const int s = row_ptr[row0 + b];
    const int len = max(0, min(row_ptr[row0 + b + 1] - s, nb));
    for (int p = 0; p < len; ++p) {
      const int kb = col_idx[s + p];
      if (kb >= 0 && kb < nb) row[kb >> 5] |= 1u << (kb & 31);  // this thread's row only
    }
  }
  __syncthreads();
  // Threads kCandSplit*q .. kCandSplit*q + kCandSplit-1 (adjacent lanes) share block
  // i = c0 + q; thread `part` takes the partners at distances part+1, part+1+kCandSplit, ...
  const int i = c0 + tid / kCandSplit, part = tid % kCandSplit;
  uint32_t key[kPairCands];
#pragma unroll
  for (int c = 0; c < kPairCands; ++c) key[c] = 0u;
  if (i < nb) {
    uint32_t bi[kMaxWords];
#pragma unroll
    for (int w = 0; w < kMaxWords; ++w) bi[w] = w < words ? pair_bits[static_cast<size_t>(i - base) * row_words + w] : 0u;
    const int reach = min(kPairWindow, max(i, nb - 1 - i));
    for (int dd = part + 1; dd <= reach; dd += kCandSplit) {
#pragma unroll
      for (int side = 0; side < 2; ++side) {
        const int j = side == 0 ? i - dd : i + dd;
        if (j >= 0 && j < nb) {
          const uint32_t* bj = pair_bits + static_cast<size_t>(j - base) * row_words;
          int ov = 0;
#pragma unroll
          for (int w = 0; w < kMaxWords; ++w)
            if (w < words) ov += __popc(bi[w] & bj[w]);
          pair_insert(key, pair_key(ov, dd, side));
        }
      }
    }
  }
  // Merge the lists of the threads sharing block i (keys are distinct, so the result does
  // not depend on how the window was split).
#pragma unroll
  for (int m = 1; m < kCandSplit; m <<= 1) {
    uint32_t other[kPairCands];
#pragma unroll
    for (int c = 0; c < kPairCands; ++c) other[c] = __shfl_xor_sync(0xffffffffu, key[c], m);
#pragma unroll
    for (int c = 0; c < kPairCands; ++c) pair_insert(key, other[c]);
  }
  if (i < nb && part == 0) {
    int16_t* out = cand + (row0 + i) * kPairCands;
#pragma unroll
    for (int c = 0; c < kPairCands; ++c) out[c] = static_cast<int16_t>(pair_key_block(key[c], i));
  }
}

// Steps 2 and 3.  grid (B*H), kPairThreads threads, pair_match_smem_bytes(n_blocks)
// dynamic shared memory (none at block size 128, where cand is not read).
// tile_blocks: int32 [B*H][n_tiles][2].
__global__ void __launch_bounds__(kPairThreads)
    pair_match_kernel(const int16_t* __restrict__ cand_g, int n_blocks, int n_tiles, int bs,
                      int32_t* __restrict__ tile_blocks) {
  extern __shared__ int16_t pair_match_smem[];
  __shared__ int skip;
  if (threadIdx.x == 0) skip = device_status_set() ? 1 : 0;
  __syncthreads();
  if (skip) return;  // an earlier kernel failed (block-uniform)
  const int bh = blockIdx.x, tid = threadIdx.x;
  const int nb = n_blocks;
  int32_t* out = tile_blocks + static_cast<size_t>(bh) * n_tiles * 2;
  if (bs != 64) {
    for (int t = tid; t < n_tiles; t += kPairThreads) {
      out[2 * t] = t < nb ? t : -1;
      out[2 * t + 1] = -1;
    }
    return;
  }
  int16_t* cand = pair_match_smem;  // [nb][kPairCands]
  int16_t* partner = cand + static_cast<size_t>(nb) * kPairCands;
  int16_t* choice = partner + nb;
  const int16_t* cg = cand_g + static_cast<size_t>(bh) * nb * kPairCands;
  for (int x = tid; x < nb * kPairCands; x += kPairThreads) cand[x] = cg[x];
  for (int x = tid; x < nb; x += kPairThreads) partner[x] = -1;
  __syncthreads();

  // 2. mutual choice
  for (int round = 0; round < kPairRounds; ++round) {
    for (int i = tid; i < nb; i += kPairThreads) {
      int pick = -1;
      if (partner[i] < 0) {
        for (int c = 0; c < kPairCands; ++c) {
          const int j = cand[i * kPairCands + c];
          if (j >= 0 && partner[j] < 0) {
            pick = j;
            break;
          }
        }
      }
      choice[i] = static_cast<int16_t>(pick);
    }
    __syncthreads();
    for (int i = tid; i < nb; i += kPairThreads) {
      const int j = choice[i];
      if (j > i && choice[j] == i) {
        partner[i] = static_cast<int16_t>(j);
        partner[j] = static_cast<int16_t>(i);
      }
    }
    __syncthreads();
  }

  // 3. tiles, written by warp 0 with ballot scans
  if (tid < 32) {
    const int lane = tid;
    int t = 0;
    for (int b0 = 0; b0 < nb; b0 += 32) {
      const int i = b0 + lane;
      const int p = i < nb ? partner[i] : -1;
      const bool low = p > i;
      const uint32_t m = __ballot_sync(0xffffffffu, low);
      if (low) {
        const int at = t + __popc(m & ((1u << lane) - 1u));
        out[2 * at] = i;
        out[2 * at + 1] = p;
      }
      t += __popc(m);
    }
    int left = 0;  // unpaired blocks placed so far
    for (int b0 = 0; b0 < nb; b0 += 32) {
      const int i = b0 + lane;
      const bool alone = i < nb && partner[i] < 0;
      const uint32_t m = __ballot_sync(0xffffffffu, alone);
      if (alone) {
        const int k = left + __popc(m & ((1u << lane) - 1u));
        out[2 * (t + k / 2) + (k & 1)] = i;
      }
      left += __popc(m);
    }
    if (lane == 0 && (left & 1)) out[2 * (t + left / 2) + 1] = -1;
  }
}

}  // namespace rt
