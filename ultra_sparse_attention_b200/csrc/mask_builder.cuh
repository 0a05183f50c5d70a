// mask_builder.cuh -- which key blocks each query block keeps.
//
// Re-ttention project page, Abstract: the sparse step attends to a small
// subset of the tokens (down to 3.1% of them).  The subset rule used here:
// mean-pool each block of Q and K, score every (query block, key block) pair
// by the scaled dot product of the pooled vectors, keep the forced prefix
// blocks plus the best-scoring others, ties to the lower block index, and
// emit the kept set sorted ascending as a CSR row.
//
// Two kernels, both bound by memory or latency, not by arithmetic:
//   pool_blocks_kernel   reads Q and K once (HBM-bound), writes fp32 block
//                        means [BH, n_blocks, D] (pad columns zero);
//   score_select_kernel  eight query blocks per CTA: their scores against every
//                        key block (pooled K staged in shared memory, each
//                        thread scoring one key block against four query
//                        blocks), then one warp per query block selects the
//                        top k in the (score desc, index asc) order -- up to 8
//                        by rounds of a warp arg-max, more by a threshold found
//                        with a binary search over order-preserving score keys
//                        -- and a ballot scan writes the row ascending.
//   mass_select_kernel   the same selection on exact block attention masses.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace rt {

constexpr int kPoolRowGroups = 16;

// grid (n_blocks, B*H, 2): z = 0 pools Q, z = 1 pools K.  D/8 * 16 threads.
template <int D>
__global__ void __launch_bounds__(D / 8 * kPoolRowGroups)
    pool_blocks_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, int N, int d,
                       int bs, float* __restrict__ pooled_q, float* __restrict__ pooled_k) {
  constexpr int kChunks = D / 8;  // 16-byte chunks per row
  __shared__ float partial[kPoolRowGroups][D];
  __shared__ int skip;
  if (threadIdx.x == 0) skip = device_status_set() ? 1 : 0;
  __syncthreads();
  if (skip) return;  // an earlier kernel failed (block-uniform)
  const int b = blockIdx.x, bh = blockIdx.y;
  const __nv_bfloat16* x = blockIdx.z == 0 ? q : k;
  float* out = blockIdx.z == 0 ? pooled_q : pooled_k;
  const int n_blocks = gridDim.x;
  const int row0 = b * bs;
  const int count = min(bs, N - row0);
  const int t = threadIdx.x;
  const int ch = t % kChunks, rg = t / kChunks;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const uint4* base = reinterpret_cast<const uint4*>(x + (static_cast<size_t>(bh) * N + row0) * D) + ch;
  for (int r = rg; r < count; r += kPoolRowGroups) {
    uint4 u = __ldg(base + static_cast<size_t>(r) * kChunks);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += bf16_lo_to_f32(w[i]);
      acc[2 * i + 1] += bf16_hi_to_f32(w[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) partial[rg][ch * 8 + i] = acc[i];
  __syncthreads();
  for (int c = t; c < D; c += blockDim.x) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < kPoolRowGroups; ++g) s += partial[g][c];
    out[(static_cast<size_t>(bh) * n_blocks + b) * D + c] = c < d ? s / static_cast<float>(count) : 0.f;
  }
}

constexpr int kSelWarps = 8;      // query blocks per CTA
constexpr int kSelChunk = 128;    // key blocks staged in shared memory at a time

__host__ __device__ constexpr int select_words(int n_blocks) { return (n_blocks + 31) / 32; }

// Pooled rows in shared memory are D + 4 floats apart: 16-byte aligned for 128-bit loads, and
// eight consecutive rows (one phase of a warp's 128-bit access) fall on distinct banks.
template <int D>
__host__ __device__ constexpr int sel_stride() { return D + 4; }

template <int D>
__host__ __device__ constexpr size_t score_select_smem_bytes(int n_blocks) {
  return sizeof(float) * (static_cast<size_t>(kSelChunk) * sel_stride<D>() + kSelWarps * D +
                          static_cast<size_t>(kSelWarps) * n_blocks) +
         sizeof(uint32_t) * kSelWarps * select_words(n_blocks);
}

// Up to this many blocks are chosen by rounds of a warp arg-max; more by a threshold.
constexpr int kSelRoundsMax = 8;

// Unsigned key with the order of the float scores (-inf lowest; NaN never reaches here).
__device__ __forceinline__ uint32_t order_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// (score, index) order of the selection: higher score first, lower index on ties.
__device__ __forceinline__ bool sel_better(float sa, int ka, float sb, int kb) {
  return sa > sb || (sa == sb && ka < kb);
}

// One query block's selection by a warp: the top `keep` key blocks of my_sc[0, n_blocks) in the
// (score desc, index asc) order, the forced prefix blocks first -- up to 8 by rounds of a warp
// arg-max, more by a threshold found with a binary search over order-preserving score keys --
// then a ballot scan that writes CSR row `row` ascending (row_ptr[row], and row_ptr[row + 1]
// for the last row).  my_taken: select_words(n_blocks) words of scratch, cleared here.
__device__ __forceinline__ void select_row(const float* my_sc, uint32_t* my_taken, int n_blocks, int bs, int keep,
                                           int forced_tokens, size_t row, bool last_row,
                                           int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx,
                                           int lane) {
  const int words = select_words(n_blocks);
  for (int w = lane; w < words; w += 32) my_taken[w] = 0u;
  __syncwarp();
  const int forced = min(n_blocks, forced_tokens > 0 ? (forced_tokens + bs - 1) / bs : 0);
  for (int kb = lane; kb < forced; kb += 32) atomicOr(&my_taken[kb / 32], 1u << (kb % 32));
  __syncwarp();
  const int need = keep - forced;  // blocks to choose among kb >= forced
  if (need > kSelRoundsMax) {
    // Threshold selection: T = the need-th largest order key among the candidates (a binary
    // search over the 32 key bits, one warp count per bit), then every candidate above T and
    // the lowest-index candidates equal to T.  Same set as `need` rounds of the arg-max.
    uint32_t T = 0u;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      int c = 0;
      for (int kb = forced + lane; kb < n_blocks; kb += 32) c += order_key(my_sc[kb]) >= cand ? 1 : 0;
      if (static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<uint32_t>(c))) >= need) T = cand;
    }
    int gt = 0;
    for (int kb = forced + lane; kb < n_blocks; kb += 32) gt += order_key(my_sc[kb]) > T ? 1 : 0;
    int ties_left = need - static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<uint32_t>(gt)));
    for (int base = forced; base < n_blocks; base += 32) {
      const int kb = base + lane;
      const bool in = kb < n_blocks;
      const uint32_t key = in ? order_key(my_sc[kb]) : 0u;
      const bool tie = in && key == T;
      const uint32_t tmask = __ballot_sync(0xffffffffu, tie);
      const int before = __popc(tmask & ((1u << lane) - 1u));
      if (in && (key > T || (tie && before < ties_left))) atomicOr(&my_taken[kb / 32], 1u << (kb % 32));
      ties_left -= __popc(tmask);
    }
    __syncwarp();
  }
  for (int round = need > kSelRoundsMax ? keep : forced; round < keep; ++round) {
    float best_s = -INFINITY;
    int best_k = n_blocks;  // sentinel: loses to every real block
    for (int kb = forced + lane; kb < n_blocks; kb += 32) {
      if ((my_taken[kb / 32] >> (kb % 32)) & 1u) continue;
      const float s = my_sc[kb];
      if (sel_better(s, kb, best_s, best_k)) { best_s = s; best_k = kb; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, best_s, off);
      const int ok = __shfl_xor_sync(0xffffffffu, best_k, off);
      if (sel_better(os, ok, best_s, best_k)) { best_s = os; best_k = ok; }
    }
    if (lane == 0 && best_k < n_blocks) my_taken[best_k / 32] |= 1u << (best_k % 32);
    __syncwarp();
  }

  int32_t* out = col_idx + row * keep;
  int written = 0;
  for (int base = 0; base < n_blocks; base += 32) {
    const int kb = base + lane;
    const bool t = kb < n_blocks && ((my_taken[kb / 32] >> (kb % 32)) & 1u);
    const uint32_t mask = __ballot_sync(0xffffffffu, t);
    const int pos = written + __popc(mask & ((1u << lane) - 1u));
    if (t && pos < keep) out[pos] = kb;
    written += __popc(mask);
  }
  if (lane == 0) {
    row_ptr[row] = static_cast<int32_t>(row * keep);
    if (last_row) row_ptr[row + 1] = static_cast<int32_t>((row + 1) * keep);
  }
}

// grid (ceil(n_blocks / kSelWarps), B*H), 32*kSelWarps threads.
template <int D>
__global__ void __launch_bounds__(32 * kSelWarps)
    score_select_kernel(const float* __restrict__ pooled_q, const float* __restrict__ pooled_k, int n_blocks,
                        int bs, float scale, int keep, int forced_tokens, int32_t* __restrict__ row_ptr,
                        int32_t* __restrict__ col_idx, float* __restrict__ block_scores) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  constexpr int kS = sel_stride<D>();
  static_assert(D % 4 == 0, "pooled rows are read as float4");
  float* pk = reinterpret_cast<float*>(smem_raw);                 // [kSelChunk][D+4]
  float* pq = pk + kSelChunk * kS;                                // [kSelWarps][D]
  float* sc = pq + kSelWarps * D;                                 // [kSelWarps][n_blocks]
  uint32_t* taken = reinterpret_cast<uint32_t*>(sc + kSelWarps * n_blocks);  // [kSelWarps][words]
  __shared__ int skip;
  if (threadIdx.x == 0) skip = device_status_set() ? 1 : 0;
  __syncthreads();
  if (skip) return;  // an earlier kernel failed (block-uniform)

  const int bh = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qb = blockIdx.x * kSelWarps + warp;
  const bool have_row = qb < n_blocks;
  const int words = select_words(n_blocks);
  const size_t head = static_cast<size_t>(bh) * n_blocks;

  for (int i = threadIdx.x; i < kSelWarps * (D / 4); i += blockDim.x) {
    const int w = i / (D / 4), c4 = i % (D / 4);
    const int qq = blockIdx.x * kSelWarps + w;
    reinterpret_cast<float4*>(pq + w * D)[c4] =
        qq < n_blocks ? reinterpret_cast<const float4*>(pooled_q + (head + qq) * D)[c4] : make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // Thread t scores key block t % kSelChunk of each staged chunk against four of the CTA's query
  // blocks, 4 * (t / kSelChunk) .. +3: one pooled K row read from shared memory serves four dot
  // products (the query rows are the same for the whole warp, a broadcast).
  static_assert(kSelWarps == 8 && kSelChunk * 2 == 32 * kSelWarps, "two groups of four query blocks");
  const int kbl = threadIdx.x % kSelChunk, q0 = 4 * (threadIdx.x / kSelChunk);
  float* my_sc = sc + warp * n_blocks;
  for (int kb0 = 0; kb0 < n_blocks; kb0 += kSelChunk) {
    __syncthreads();
    const int nch = min(kSelChunk, n_blocks - kb0);
    for (int i = threadIdx.x; i < nch * (D / 4); i += blockDim.x) {
      const int r = i / (D / 4), c4 = i % (D / 4);
      reinterpret_cast<float4*>(pk + r * kS)[c4] = reinterpret_cast<const float4*>(pooled_k + (head + kb0 + r) * D)[c4];
    }
    __syncthreads();
    if (kbl < nch) {
      const float4* b = reinterpret_cast<const float4*>(pk + kbl * kS);
      // Two FMA chains per query block keep eight chains in flight.
      float acc[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
      for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 y = b[c4];
#pragma unroll
        for (int qi = 0; qi < 4; ++qi) {
          const float4 x = reinterpret_cast<const float4*>(pq + (q0 + qi) * D)[c4];
          acc[qi][0] = fmaf(x.x, y.x, acc[qi][0]);
          acc[qi][1] = fmaf(x.y, y.y, acc[qi][1]);
          acc[qi][0] = fmaf(x.z, y.z, acc[qi][0]);
          acc[qi][1] = fmaf(x.w, y.w, acc[qi][1]);
        }
      }
#pragma unroll
      for (int qi = 0; qi < 4; ++qi) {
        if (blockIdx.x * kSelWarps + q0 + qi >= n_blocks) continue;
        float s = scale * (acc[qi][0] + acc[qi][1]);
        if (s != s) s = -INFINITY;  // a NaN never wins
        sc[(q0 + qi) * n_blocks + kb0 + kbl] = s;
      }
    }
  }
  __syncthreads();  // each row's scores were written by other threads
  if (!have_row) return;
  const size_t row = head + qb;
  select_row(my_sc, taken + warp * words, n_blocks, bs, keep, forced_tokens, row,
             row + 1 == static_cast<size_t>(gridDim.y) * n_blocks, row_ptr, col_idx, lane);
  if (block_scores != nullptr)
    for (int kb = lane; kb < n_blocks; kb += 32) block_scores[row * n_blocks + kb] = my_sc[kb];
}

// Exact-mass selection.  block_lse [B*H][n_tiles][N] holds, per key tile of 64 keys and row i,
// log2 of the row's exponential sum over the tile in the units of s*scale*log2(e); with the
// row's log-sum-exp lse2_i = m_i*log2(e) + log2(Z_full_i) (m natural, from the same pass)
//   mass[qb][kb] = sum over rows i of qb, tiles t of kb of 2^(block_lse[t][i] - lse2_i),
// the softmax probability the block's rows give the key block.  One warp per query block:
// the masses go to shared memory, then select_row keeps the largest.  grid
// (ceil(n_blocks / kSelWarps), B*H), 32*kSelWarps threads.
__host__ __device__ constexpr size_t mass_select_smem_bytes(int n_blocks) {
  return sizeof(float) * static_cast<size_t>(kSelWarps) * n_blocks +
         sizeof(uint32_t) * kSelWarps * select_words(n_blocks);
}

__global__ void __launch_bounds__(32 * kSelWarps)
    mass_select_kernel(const float* __restrict__ block_lse, const float* __restrict__ stat_m,
                       const float* __restrict__ stat_zfull, int N, int n_blocks, int bs, int keep,
                       int forced_tokens, int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx,
                       float* __restrict__ block_mass) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* sc = reinterpret_cast<float*>(smem_raw);                            // [kSelWarps][n_blocks]
  uint32_t* taken = reinterpret_cast<uint32_t*>(sc + kSelWarps * n_blocks);  // [kSelWarps][words]
  __shared__ int skip;
  if (threadIdx.x == 0) skip = device_status_set() ? 1 : 0;
  __syncthreads();
  if (skip) return;  // an earlier kernel failed (block-uniform)
  const int bh = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qb = blockIdx.x * kSelWarps + warp;
  if (qb >= n_blocks) return;  // no block-wide synchronisation below
  const int n_tiles = (N + 63) / 64;
  const int tiles_per_block = bs / 64;
  const int i0 = qb * bs;
  // Up to four rows per lane (block size 128): their log-sum-exp in log2 units.
  float lse2[4];
  int rows[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int r = lane + 32 * t;
    rows[t] = (r < bs && i0 + r < N) ? i0 + r : -1;
    lse2[t] = 0.f;
    if (rows[t] >= 0) {
      const size_t g = static_cast<size_t>(bh) * N + rows[t];
      lse2[t] = __ldg(stat_m + g) * 1.4426950408889634f + __log2f(__ldg(stat_zfull + g));
    }
  }
  float* my_sc = sc + warp * n_blocks;
#pragma unroll 4
  for (int kb = 0; kb < n_blocks; ++kb) {
    float acc = 0.f;
    for (int tt = 0; tt < tiles_per_block; ++tt) {
      const int kt = kb * tiles_per_block + tt;
      if (kt >= n_tiles) break;
      const float* src = block_lse + (static_cast<size_t>(bh) * n_tiles + kt) * N;
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (rows[t] >= 0) acc += ex2_approx(__ldg(src + rows[t]) - lse2[t]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) my_sc[kb] = acc;
  }
  __syncwarp();
  const size_t row = static_cast<size_t>(bh) * n_blocks + qb;
  select_row(my_sc, taken + warp * select_words(n_blocks), n_blocks, bs, keep, forced_tokens, row,
             row + 1 == static_cast<size_t>(gridDim.y) * n_blocks, row_ptr, col_idx, lane);
  if (block_mass != nullptr)
    for (int kb = lane; kb < n_blocks; kb += 32) block_mass[row * n_blocks + kb] = my_sc[kb];
}

}  // namespace rt
