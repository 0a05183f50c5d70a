// attention.cuh -- the two attention kernels of Re-ttention on tcgen05 tensor cores.
//
//   full_capture_kernel    full attention at a capture step; per row it also
//                          emits the statistics the later sparse steps reuse:
//                          the reference m (the row max, lowered on rows led by
//                          masked keys so Z_kept stays in fp32), Z_full, Z_kept
//                          and the residual numerator U of the masked-out keys
//                          (project page,
//                          mechanism highlight: the ratio of the two softmax
//                          denominators, sparse over full, is reused, and what
//                          the masked keys add to the output is cached).
//   sparse_reshape_kernel  attention over the kept key blocks only, then the
//                          reshape o = (N' + e^{m_c - m'} U) / (Z' * Z_full / Z_kept)
//                          in the epilogue (teaser: sparse attention reshaped with
//                          statistics cached across denoising steps).
//
// Shared design (a 128-row query tile of one (batch, head) at a time):
//  * warp 0 issues TMA loads, warp 1 issues tcgen05.mma (the two swapped in the
//    second of two CTAs on an SM), warps 2..5 own one query row per thread
//    (TMEM lane = row) for the softmax and the epilogue.
//  * S = Q K^T lands in TMEM; the softmax writes P (bf16 in the sparse step, f16
//    scaled by 2^7 in the capture) back into the first 32 columns of the same
//    buffer and the PV product reads A = P straight from TMEM (no shared-memory
//    round trip).  The capture computes one exponential pair in eight on the
//    FMA pipe (f2_exp2_poly), the rest on the MUFU.
//  * With 64-token blocks the 128-row tile holds two query blocks, each with
//    its own kept list; the sparse kernel walks the union of both lists and a
//    row whose block does not keep a tile writes P = 0 for it.  (An M = 64 MMA
//    per query block would halve the tensor rate; the union costs only the
//    blocks the two lists do not share, and the sparse step takes its pairs
//    of query blocks from a table that pairs blocks with similar lists, see
//    pairing.cuh.)
//  * Head dim 128 is two 64-column tiles with 128-byte swizzle.
//  * Online softmax in base 2 (x = s * scale * log2 e) with a lazy reference:
//    O is rescaled only when the row max moves up by more than 8 (or down by
//    more than 64 in the sparse step, whose reference starts at the cached
//    max), so the rescale path practically never runs.
//  * Head dim 64 uses 128-byte swizzled tiles; head dim 80 adds a 16-column
//    tail tile with 32-byte swizzle (one more K-step for QK^T, one N=16 MMA for PV).
//  * Every barrier wait is bounded (see ptx.cuh) and its outcome is made
//    warp-uniform; on a timeout the block stops, drains its own copies and
//    MMAs, frees TMEM and returns.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace rt {

constexpr int kBM = 128;            // query rows per tile (tcgen05 M)
constexpr int kBN = 64;             // keys per tile
constexpr int kAttnThreads = 192;   // 6 warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleUp = 8.f;    // log2 units
constexpr float kRescaleDown = 64.f; // log2 units
constexpr float kSumUp = 0x1p8f;      // 2^kRescaleUp
constexpr float kSumDown = 0x1p-64f;  // 2^-kRescaleDown
constexpr float kPBias = 7.f;         // capture: f16 P carries p * 2^7 (p <= 2^8, so <= 2^15)
constexpr float kCacheShiftBelow = 64.f;  // capture: Z_kept below 2^-64 of the row max moves the cache reference
constexpr int kCacheShiftMax = 100;       // ... by at most 2^100 (Z_full <= 2^114.2, U <= 2^114.2 max|v|)
constexpr uint64_t kDrainLimitNs = 200000000ull;

// Tile byte sizes for head dim D (bf16 Q/K/V tiles).  A tile is its 64-column
// main part (128-byte rows, 128-byte swizzle) followed, for D > 64, by a tail
// part: 16 columns (32-byte rows, 32-byte swizzle) for D = 80, another 64
// columns laid out like the main part for D = 128.
template <int D>
struct Tiles {
  static_assert(D == 64 || D == 80 || D == 128, "head_dim_padded must be 64, 80 or 128");
  static constexpr int kTailCols = D - 64;
  static constexpr bool kTail = kTailCols > 0;
  static constexpr bool kTailWide = kTailCols == 64;
  static constexpr int kTailRow = kTailCols * 2;                          // bytes per tail row
  static constexpr uint32_t kTailSwizzle = kTailWide ? kSwizzle128B : kSwizzle32B;
  static constexpr int kTailSBO = 8 * kTailRow;                           // 8-row group stride
  static constexpr int kTailKSteps = kTailCols / 16;
  static constexpr int kQMain = kBM * 128;
  static constexpr int kQTail = kBM * kTailRow;
  static constexpr int kQBytes = kQMain + kQTail;
  static constexpr int kKVMain = kBN * 128;
  static constexpr int kKVTail = kBN * kTailRow;
  static constexpr int kKVBytes = kKVMain + kKVTail;   // one K or one V tile
  static constexpr int kStageBytes = 2 * kKVBytes;     // K tile then V tile
  static constexpr int kKSteps = D / 16;
  // PV into the tail columns of the accumulator: N = the tail's width.
  static constexpr uint32_t kIdescPVTail = idesc_bf16(kBM, kTail ? kTailCols : 16, false, true);
  static constexpr uint32_t kIdescPVTailF16 = idesc_f16(kBM, kTail ? kTailCols : 16, false, true);
};

struct AttnArgs {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  // sparse step: cached statistics (all null = plain block-sparse attention)
  const float* stat_m;
  const float* stat_zfull;
  const float* stat_zkept;
  const float* stat_u;
  // compressed cache: U as f16 bits [B*H, N, D] times a per-row power of two (fp32 [B*H, N])
  const uint16_t* stat_u16;
  const float* stat_u_scale;
  // capture step: statistics out
  float* out_m;
  float* out_zfull;
  float* out_zkept;
  float* out_u;
  uint16_t* out_u16;     // compressed cache out (instead of out_u)
  float* out_u_scale;
  // capture step, optional: per 64-key tile t and row i, log2 of the row's exponential sum over
  // the tile (units of s * scale * log2 e), fp32 [B*H][ceil(N/64)][N]
  float* out_block_lse;
  __nv_bfloat16* out;
  // sparse step: the query blocks of each 128-row tile, int32 [B*H][n_tiles][2]
  // (-1: empty half); null = the neighbouring blocks
  const int32_t* tile_blocks;
  // capture step: per (batch, head) the bits of max |v|, which fix the power-of-two scale
  // of the f16 copy of V (see v_scale_exp)
  const uint32_t* v_amax;
  int N;
  int d;
  int n_blocks;
  int n_heads;       // B*H
  float scale_log2;  // softmax scale * log2(e)
};

// Power-of-two exponent k of the capture's f16 copy of V for a head whose max |v| has the
// float bits `amax`: max |v| * 2^k lies in [2^14, 2^15), well inside f16 (max 65504), so
// every finite bf16 value down to 2^-30 of the head's largest keeps 11 mantissa bits.  A
// head of zeros or with a non-finite max is not scaled.  k in [-113, 126] keeps 2^k normal.
__host__ __device__ constexpr int v_scale_exp(uint32_t amax) {
  return (((amax >> 23) & 0xFFu) == 0xFFu || amax == 0u)
             ? 0
             : (14 - (static_cast<int>((amax >> 23) & 0xFFu) - 127) > 126 ? 126
                                                                         : 14 - (static_cast<int>((amax >> 23) & 0xFFu) - 127));
}

__device__ __forceinline__ float exp2_int(int k) {  // 2^k for k in [-126, 127]
  return __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
}

__host__ __device__ constexpr int attn_words(int n_blocks) { return (n_blocks + 31) / 32; }
__host__ __device__ constexpr int key_tiles(int N) { return (N + kBN - 1) / kBN; }
__host__ __device__ constexpr int query_tiles(int N) { return (N + kBM - 1) / kBM; }

// ------------------------------------------------------------------ MMA issue
constexpr uint32_t kIdescQK = idesc_bf16(kBM, kBN, false, false);
constexpr uint32_t kIdescPV64 = idesc_bf16(kBM, 64, false, true);
constexpr uint32_t kIdescPV64F16 = idesc_f16(kBM, 64, false, true);  // capture: f16 P and f16 V

// S = Q K^T for one key tile into TMEM at `s_tmem`, Q and K in shared memory.
// The issue helpers below are warp-collective (one elected lane issues).  The
// descriptors are built once and advanced by adding to their start-address
// field (16-byte units).
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint32_t q_base, uint32_t k_base) {
  const uint64_t qd = smem_desc(q_base, 16, 1024, kSwizzle128B);
  const uint64_t kd = smem_desc(k_base, 16, 1024, kSwizzle128B);
  mma_ss_w(s_tmem, qd, kd, kIdescQK, 0u);
#pragma unroll
  for (int ks = 1; ks < 4; ++ks) mma_ss_w(s_tmem, qd + 2 * ks, kd + 2 * ks, kIdescQK, 1u);
  if constexpr (Tiles<D>::kTail) {
    using T = Tiles<D>;
    const uint64_t qt = smem_desc(q_base + T::kQMain, 16, T::kTailSBO, T::kTailSwizzle);
    const uint64_t kt = smem_desc(k_base + T::kKVMain, 16, T::kTailSBO, T::kTailSwizzle);
#pragma unroll
    for (int ks = 0; ks < T::kTailKSteps; ++ks) mma_ss_w(s_tmem, qt + 2 * ks, kt + 2 * ks, kIdescQK, 1u);
  }
}

// The same with Q resident in TMEM (D/2 columns of bf16 pairs): only K is
// read from shared memory, which keeps an N = 64 tile at the full MMA rate
// (with both operands in shared memory it is bound by the shared-memory
// bandwidth: 6 KB per 32-cycle MMA).
template <int D>
__device__ __forceinline__ void issue_qk_tq(uint32_t s_tmem, uint32_t q_tmem, uint32_t k_base) {
  const uint64_t kd = smem_desc(k_base, 16, 1024, kSwizzle128B);
  mma_ts_w(s_tmem, q_tmem, kd, kIdescQK, 0u);
#pragma unroll
  for (int ks = 1; ks < 4; ++ks) mma_ts_w(s_tmem, q_tmem + ks * 8, kd + 2 * ks, kIdescQK, 1u);
  static_assert(!Tiles<D>::kTail, "Q in TMEM is used for head dim 64 only");
}

// Copy a 128-row bf16 Q tile (K-major: 128-byte swizzled main part, 32-byte
// swizzled tail for D = 80) into D/2 TMEM columns.
template <int D>
__device__ __forceinline__ void copy_q_to_tmem(uint32_t q_tmem, uint32_t q_base) {
  const uint64_t qd = smem_desc(q_base, 16, 1024, kSwizzle128B);
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) tmem_cp_128x256b_w(q_tmem + ks * 8, qd + 2 * ks);
  static_assert(!Tiles<D>::kTail, "Q in TMEM is used for head dim 64 only");
}

// acc (+)= P V for one key tile; P is in TMEM at `p_tmem` (32 columns), bf16 with bf16 V,
// or f16 with f16 V when kF16 (the capture kernel).
template <int D, bool kF16 = false>
__device__ __forceinline__ void issue_pv(uint32_t acc_tmem, uint32_t p_tmem, uint32_t v_base, bool accumulate) {
  constexpr uint32_t kId = kF16 ? kIdescPV64F16 : kIdescPV64;
  constexpr uint32_t kIdTail = kF16 ? Tiles<D>::kIdescPVTailF16 : Tiles<D>::kIdescPVTail;
  const uint64_t vd = smem_desc(v_base, Tiles<D>::kKVMain, 1024, kSwizzle128B);
  const uint32_t acc0 = accumulate ? 1u : 0u;
  mma_ts_w(acc_tmem, p_tmem, vd, kId, acc0);
#pragma unroll
  for (int ks = 1; ks < kBN / 16; ++ks) mma_ts_w(acc_tmem, p_tmem + ks * 8, vd + 128 * ks, kId, 1u);
  if constexpr (Tiles<D>::kTail) {
    using T = Tiles<D>;
    const uint64_t vt = smem_desc(v_base + T::kKVMain, T::kKVTail, T::kTailSBO, T::kTailSwizzle);
    mma_ts_w(acc_tmem + 64, p_tmem, vt, kIdTail, acc0);
#pragma unroll
    for (int ks = 1; ks < kBN / 16; ++ks) mma_ts_w(acc_tmem + 64, p_tmem + ks * 8, vt + T::kTailRow * ks, kIdTail, 1u);
  }
}

template <int D>
__device__ __forceinline__ void load_q(unsigned char* dst, const CUtensorMap* tq, const CUtensorMap* tq_tail,
                                       uint64_t* bar, int row0, int bh) {
  mbar_arrive_expect_tx(bar, Tiles<D>::kQBytes);
  tma_load_3d(dst, tq, bar, 0, row0, bh);
  if constexpr (Tiles<D>::kTail) tma_load_3d(dst + Tiles<D>::kQMain, tq_tail, bar, 64, row0, bh);
}

// One 64-key K or V tile (main + tail) into `dst`, completing on `bar`.
template <int D>
__device__ __forceinline__ void load_kv_tile(unsigned char* dst, const CUtensorMap* t, const CUtensorMap* t_tail,
                                             uint64_t* bar, int row0, int bh) {
  mbar_arrive_expect_tx(bar, Tiles<D>::kKVBytes);
  tma_load_3d(dst, t, bar, 0, row0, bh);
  if constexpr (Tiles<D>::kTail) tma_load_3d(dst + Tiles<D>::kKVMain, t_tail, bar, 64, row0, bh);
}

// K then V tile of one key tile into a combined stage, completing on one barrier.
template <int D>
__device__ __forceinline__ void load_kv(unsigned char* stage, const CUtensorMap* tk, const CUtensorMap* tk_tail,
                                        const CUtensorMap* tv, const CUtensorMap* tv_tail, uint64_t* bar, int row0,
                                        int bh) {
  using T = Tiles<D>;
  mbar_arrive_expect_tx(bar, T::kStageBytes);
  tma_load_3d(stage, tk, bar, 0, row0, bh);
  if constexpr (T::kTail) tma_load_3d(stage + T::kKVMain, tk_tail, bar, 64, row0, bh);
  tma_load_3d(stage + T::kKVBytes, tv, bar, 0, row0, bh);
  if constexpr (T::kTail) tma_load_3d(stage + T::kKVBytes + T::kKVMain, tv_tail, bar, 64, row0, bh);
}

// ------------------------------------------------------------------ softmax helpers
// Bounded wait whose outcome is the same for every lane of the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// Rescale NCOLS fp32 columns of this thread's TMEM row by f (warp-collective).
template <int NCOLS>
__device__ __forceinline__ void tmem_row_scale(uint32_t taddr, float f) {
#pragma unroll
  for (int c0 = 0; c0 < NCOLS; c0 += 16) {
    float v[16];
    tmem_ld16(taddr + c0, v);
    uint32_t r[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(v[i] * f);
    tmem_st16(taddr + c0, r);
  }
  tmem_st_wait();
}

__device__ __forceinline__ void tmem_st32_zero(uint32_t taddr) {
  const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  tmem_st16(taddr, z);
  tmem_st16(taddr + 16, z);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&pk)[32]) {
  tmem_st16(taddr, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
  tmem_st16(taddr + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
}

// Mask key columns at or beyond N (only the ragged last tile has any).
__device__ __forceinline__ void mask_tail(float (&s)[64], int key0, int N) {
  if (key0 + kBN > N) {
#pragma unroll
    for (int c = 0; c < 64; ++c)
      if (key0 + c >= N) s[c] = -INFINITY;
  }
}

// Row max of 64 scores: four independent 3-input max chains (short dependency depth).
__device__ __forceinline__ float row_max64(const float (&s)[64]) {
  float m[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) m[k] = fmax3(s[k], s[k + 4], s[k + 8]);
#pragma unroll
  for (int c = 12; c < 60; c += 8)
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = fmax3(m[k], s[c + k], s[c + 4 + k]);
#pragma unroll
  for (int k = 0; k < 4; ++k) m[k] = fmaxf(m[k], s[60 + k]);
  return fmax3(m[0], m[1], fmaxf(m[2], m[3]));
}

// One row's 64 scores to p = 2^(s*C - m): bf16 pairs into pk, returns their fp32 sum.
__device__ __forceinline__ float exp_row64(const float (&s)[64], float m, uint64_t C2, uint32_t (&pk)[32]) {
  const uint64_t nref = f2_pack(-m, -m);
  uint64_t zz = f2_pack(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    float x0, x1;
    f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), C2, nref), x0, x1);
    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
    zz = f2_add(zz, f2_pack(p0, p1));
    pk[c / 2] = pack_bf16x2(p0, p1);
  }
  float z0, z1;
  f2_unpack(zz, z0, z1);
  return z0 + z1;
}

// U's coefficient in the sparse epilogue, times 2^100, on a row led by masked keys:
// e^{m_c - m'} Z_kept / (Z_full Z') from logarithms, or 1 / Z_full when Z_kept is 0.  Rare, and
// kept out of line: inlined, it costs the common epilogue ~2% (register pressure at the cap).
__device__ __noinline__ float far_row_u_coef(float gap, float zk, float zf, float z) {
  return zk > 0.f ? ex2_approx(gap + __log2f(zk) - __log2f(zf) - __log2f(z) + 100.f) : __fdividef(0x1p100f, zf);
}

__device__ __forceinline__ bool bitmap_has(const uint32_t* bm, int kb) { return (bm[kb / 32] >> (kb % 32)) & 1u; }

// Set the bits of the kept key blocks of query block `qb` of head `bh` (threads `t0, t0+stride, ...`).
__device__ __forceinline__ void mark_kept_blocks(uint32_t* bm, const AttnArgs& a, int bh, int qb, int t0,
                                                 int stride) {
  if (qb < 0 || qb >= a.n_blocks) return;
  const size_t r = static_cast<size_t>(bh) * a.n_blocks + qb;
  const int s = a.row_ptr[r], e = a.row_ptr[r + 1];
  const int len = max(0, min(e - s, a.n_blocks));
  for (int i = t0; i < len; i += stride) {
    const int kb = a.col_idx[s + i];
    if (kb >= 0 && kb < a.n_blocks) atomicOr(&bm[kb / 32], 1u << (kb % 32));
  }
}

// ================================================================== sparse step (persistent)
//
// Kept key tiles of a 128-row query tile, built from the CSR in shared memory
// by the producer warp two tiles ahead: list[0] = count, list[1 + j] =
// tile << 2 | (kept by query block 0) | (kept by query block 1) << 1, the
// union of the tile's query blocks' kept lists in ascending order.
__host__ __device__ constexpr int tile_list_cap(int N) { return (key_tiles(N) + 1 + 7) / 8 * 8; }

// Query block in half h of 128-row tile qt of head bh, or -1 for none: the
// pairing table's entry when there is one (out-of-range entries read as -1),
// else the neighbouring blocks qt * (128 / BS) + h.
template <int BS>
__device__ __forceinline__ int tile_query_block(const AttnArgs& a, int n_qt, int bh, int qt, int h) {
  if (h >= kBM / BS) return -1;
  const int qb = a.tile_blocks != nullptr ? __ldg(a.tile_blocks + (static_cast<size_t>(bh) * n_qt + qt) * 2 + h)
                                          : qt * (kBM / BS) + h;
  return qb >= 0 && qb < a.n_blocks ? qb : -1;
}


// The sparse kernel.  Grid: up to two CTAs per SM, each walking query tiles
// t = blockIdx.x, blockIdx.x + gridDim.x, ... in head-major order
// (neighbouring CTAs share a head, so its K/V stay in L2).
//
// Measured on this part: a tcgen05.mma issued by an elected lane of a
// converged warp costs ~11 cycles, a commit ~50, a wait on a completed
// mbarrier ~60 and a hand-off between warps ~110-150.  The pipeline:
//  * warp 0 (producer): builds the key-tile list of tile i+2 from the CSR
//    (kept-block bitmaps and a ballot scan), and its lane 0 loads Q(i) into
//    one of two buffers, streams K(g) and V(g) of every key tile g into two
//    rings under ONE barrier per key tile, and issues the TMA store of each
//    finished tile (polled, so no warp ever waits on a store);
//  * warp 1 (MMA, warp-collective issue): at the first key tile of a query
//    tile it copies Q into TMEM (head dim 64); step g issues PV(g-2), then
//    QK^T(g), then one commit to step[g % 8] -- which tells the softmax that
//    S(g) is ready and P[g & 1] (aliased into S) was consumed, and tells the
//    producer that the K slot of g and the V slot of g-2 are free;
//  * warps 2-5 (softmax + epilogue): one row per thread; P is written as bf16
//    into the first 32 columns of S[g & 1].
// TMEM (256 columns): S0 [0,64) S1 [64,128) O [128,128+D); head dim 64 adds
// two Q buffers [192,224) [224,256), so QK^T reads only K from shared memory
// (with both operands there an N = 64 QK^T is bound by shared-memory bandwidth).
// The epilogue releases O right after reading it, combines it with U (whose
// row each thread prefetched into L2 a tile earlier), and writes bf16 rows
// into the tile's Q buffer, which the producer then stores with one TMA store.
template <int D>
struct SparseLayout {
  using T = Tiles<D>;
  static constexpr int kNK = D == 64 ? 3 : 2;  // K ring
  static constexpr int kNV = D == 64 ? 5 : 4;  // V ring
  static_assert(kNV - 2 == kNK, "K(g) and V(g) load together once step g - kNK is done");
  static constexpr int kNL = 3;                // tile-list buffers
  static constexpr int kOffQ = 0;              // two Q / output staging buffers
  static constexpr int kOffK = 2 * T::kQBytes;
  static constexpr int kOffV = kOffK + kNK * T::kKVBytes;
  static constexpr int kOffLists = kOffV + kNV * T::kKVBytes;
};

struct alignas(8) SparseShared {
  uint64_t q_full[2];
  uint64_t kv_full[8], step[8];
  uint64_t p_full[2];
  uint64_t o_full, o_empty;
  uint64_t staged[2];
  uint64_t list_full[3], list_empty[3];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  uint32_t list_bits[2 * 64];  // the producer's scratch: kept-block bitmaps of a tile's two query blocks
};

template <int D>
__host__ __device__ constexpr size_t sparse_smem_bytes(int N) {
  return 1024 + SparseLayout<D>::kOffLists + SparseLayout<D>::kNL * 2 * tile_list_cap(N) + sizeof(SparseShared);
}

template <int D, int BS, bool kU16>
__global__ void __launch_bounds__(kAttnThreads, 2)
    sparse_reshape_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tq_tail,
                          const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tk_tail,
                          const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tv_tail,
                          const __grid_constant__ CUtensorMap to, const __grid_constant__ CUtensorMap to_tail,
                          const AttnArgs a) {
  using T = Tiles<D>;
  using L = SparseLayout<D>;
  static_assert(BS == 64 || BS == 128, "block size must be 64 or 128");
  constexpr int NK = L::kNK, NV = L::kNV, NL = L::kNL;
  constexpr int kQB = kBM / BS;
  constexpr uint32_t kTmemCols = 256;
  constexpr uint32_t kOCol = 128;
  constexpr uint32_t kQCol = 192;             // head dim 64: two Q buffers of 32 columns
  constexpr bool kQTmem = D == 64;

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sbase = smem_u32(smem);
  const int cap = tile_list_cap(a.N);
  uint16_t* lists = reinterpret_cast<uint16_t*>(smem + L::kOffLists);  // [NL][cap]
  SparseShared& sh = *reinterpret_cast<SparseShared*>(smem + L::kOffLists + NL * 2 * cap);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_qt = query_tiles(a.N);
  const int n_kt = key_tiles(a.N);
  const int words = attn_words(a.n_blocks);
  const int total = n_qt * a.n_heads;
  const int n_mine = total > static_cast<int>(blockIdx.x) ? (total - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const bool has_stats = a.stat_m != nullptr;

  if (warp == 0) tmem_alloc(&sh.tmem_base, kTmemCols);
  if (threadIdx.x == 32) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.q_full[b], 1);
      mbar_init(&sh.p_full[b], 128);
      mbar_init(&sh.staged[b], 128);
    }
    for (int s = 0; s < 8; ++s) {
      mbar_init(&sh.kv_full[s], 1);
      mbar_init(&sh.step[s], 1);
    }
    for (int s = 0; s < NL; ++s) {
      mbar_init(&sh.list_full[s], 1);   // the producer, once the list is built
      mbar_init(&sh.list_empty[s], 5);  // the MMA warp + one lane of each softmax warp
    }
    mbar_init(&sh.o_full, 1);
    mbar_init(&sh.o_empty, 128);
    mbar_init(&sh.drain, 1);
    sh.abort_flag = device_status_set() ? 1 : 0;  // an earlier failure: do nothing
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  // Two CTAs share an SM, one holding TMEM columns 0-255 and the other 256-511.  The second swaps
  // the producer and MMA roles of warps 0 and 1, so that the two MMA warps sit on different SM
  // sub-partitions (a warp's sub-partition is its index mod 4) and slow different softmax warps.
  const int prod_w = (tmem & 256u) ? 1 : 0;
  volatile int* abort_flag = &sh.abort_flag;
  const bool run = sh.abort_flag == 0;  // block-uniform
  auto tile_of = [&](int i) { return static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x); };

  if (!run) {
    // an earlier kernel failed: leave the outputs untouched
  } else if (warp == prod_w) {
    // ---------------- producer (the whole warp; lane 0 issues the copies)
    int lists_built = 0, stores_issued = 0, q_loads = 0, g = 0, kslot = 0, vslot = 0;
    bool ok = true;
    uint32_t* bm = sh.list_bits;  // [2][words] scratch: the tile's query blocks' kept blocks
    // Build the key-tile list of tile `lists_built` in its buffer from the CSR; `block` waits
    // for the buffer, otherwise the call returns without building when it is still in use.
    auto build_list = [&](bool block) -> bool {
      const int i = lists_built, lb = i % NL;
      if (i >= n_mine) return true;
      if (i >= NL) {
        const uint32_t par = ((i / NL) - 1) & 1;
        if (block) {
          if (!warp_wait(&sh.list_empty[lb], par, abort_flag)) return false;
        } else if (!__all_sync(0xffffffffu, mbar_test(&sh.list_empty[lb], par))) {
          return true;
        }
      }
      const int t = tile_of(i), bh = t / n_qt, qt = t % n_qt;
      for (int w = lane; w < 2 * words; w += 32) bm[w] = 0u;
      __syncwarp();
      for (int q = 0; q < kQB; ++q)
        mark_kept_blocks(bm + q * words, a, bh, tile_query_block<BS>(a, n_qt, bh, qt, q), lane, 32);
      __syncwarp();
      uint16_t* out = lists + lb * cap;
      int count = 0;
      for (int t0 = 0; t0 < n_kt; t0 += 32) {
        const int tile = t0 + lane;
        uint32_t flags = 0u;
        if (tile < n_kt) {
          const int kb = tile * kBN / BS;
          flags = bitmap_has(bm, kb) ? 1u : 0u;
          if (kQB == 2) flags |= bitmap_has(bm + words, kb) ? 2u : 0u;
        }
        const uint32_t mask = __ballot_sync(0xffffffffu, flags != 0u);
        if (flags) out[1 + count + __popc(mask & ((1u << lane) - 1u))] = static_cast<uint16_t>((tile << 2) | flags);
        count += __popc(mask);
      }
      if (lane == 0) out[0] = static_cast<uint16_t>(count);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.list_full[lb]);
      ++lists_built;
      return true;
    };
    // Store the output of tile `stores_issued` once its epilogue has staged it.
    auto issue_store = [&](bool block) -> bool {
      const int i = stores_issued;
      const uint32_t par = (i >> 1) & 1;
      if (block) {
        if (!warp_wait(&sh.staged[i & 1], par, abort_flag)) return false;
      } else if (!__all_sync(0xffffffffu, mbar_test(&sh.staged[i & 1], par))) {
        return true;
      }
      const int t = tile_of(i), bh = t / n_qt, qt = t % n_qt;
      if (lane == 0) {
        const unsigned char* stg = smem + L::kOffQ + (i & 1) * T::kQBytes;
        // One BS-row box per query block of the tile.
#pragma unroll
        for (int h = 0; h < kQB; ++h) {
          const int qb = tile_query_block<BS>(a, n_qt, bh, qt, h);
          if (qb < 0) continue;
          tma_store_3d(&to, stg + h * BS * 128, 0, qb * BS, bh);
          if constexpr (T::kTail) tma_store_3d(&to_tail, stg + T::kQMain + h * BS * T::kTailRow, 64, qb * BS, bh);
        }
        bulk_commit_group();
      }
      ++stores_issued;
      return true;
    };
    for (int i = 0; ok && i < n_mine; ++i) {
      const int t = tile_of(i), bh = t / n_qt, qt = t % n_qt;
      while (ok && lists_built < i + 2 && lists_built < n_mine) ok = build_list(true);
      if (!ok) break;
      const int count = lists[(i % NL) * cap];  // built by this warp
      const uint16_t* lst = lists + (i % NL) * cap + 1;
      // Q(i) reuses the buffer of tile i-2 once its output store has read it.
      if (i >= 2) {
        while (ok && stores_issued <= i - 2) ok = issue_store(true);
        if (!ok) break;
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
      }
      if (lane == 0) {
        // One BS-row box per query block of the tile; an empty half is not loaded (its
        // rows keep no key tile, so their scores are never read).
        unsigned char* dst = smem + L::kOffQ + (i & 1) * T::kQBytes;
        int qb[kQB], n = 0;
#pragma unroll
        for (int h = 0; h < kQB; ++h) n += (qb[h] = tile_query_block<BS>(a, n_qt, bh, qt, h)) >= 0;
        mbar_arrive_expect_tx(&sh.q_full[i & 1], n * (T::kQBytes / kQB));
#pragma unroll
        for (int h = 0; h < kQB; ++h) {
          if (qb[h] < 0) continue;
          tma_load_3d(dst + h * BS * 128, &tq, &sh.q_full[i & 1], 0, qb[h] * BS, bh);
          if constexpr (T::kTail)
            tma_load_3d(dst + T::kQMain + h * BS * T::kTailRow, &tq_tail, &sh.q_full[i & 1], 64, qb[h] * BS, bh);
        }
      }
      ++q_loads;
      for (int j = 0; j < count; ++j, ++g) {
        if (g >= NK && !warp_wait(&sh.step[(g - NK) & 7], ((g - NK) >> 3) & 1, abort_flag)) { ok = false; break; }
        if (lane == 0) {
          const int row0 = (lst[j] >> 2) * kBN;
          uint64_t* bar = &sh.kv_full[g & 7];
          mbar_arrive_expect_tx(bar, 2 * T::kKVBytes);
          unsigned char* kd = smem + L::kOffK + kslot * T::kKVBytes;
          unsigned char* vd = smem + L::kOffV + vslot * T::kKVBytes;
          tma_load_3d(kd, &tk, bar, 0, row0, bh);
          if constexpr (T::kTail) tma_load_3d(kd + T::kKVMain, &tk_tail, bar, 64, row0, bh);
          tma_load_3d(vd, &tv, bar, 0, row0, bh);
          if constexpr (T::kTail) tma_load_3d(vd + T::kKVMain, &tv_tail, bar, 64, row0, bh);
        }
        __syncwarp();
        if (++kslot == NK) kslot = 0;
        if (++vslot == NV) vslot = 0;
        // Opportunistic work that must not wait: the next list, a finished tile's store.
        if (lists_built < n_mine) build_list(false);
        if (stores_issued < i) issue_store(false);
      }
    }
    while (ok && stores_issued < n_mine) ok = issue_store(true);
    if (lane == 0) {
      bulk_wait_group0();
      if (*abort_flag) {
        // Let every copy this block started land before the block exits.
        volatile int no_abort = 0;
        for (int i = q_loads > 2 ? q_loads - 2 : 0; i < q_loads; ++i)
          mbar_wait(&sh.q_full[i & 1], (i >> 1) & 1, &no_abort, kDrainLimitNs);
        for (int h = g > 8 ? g - 8 : 0; h < g; ++h) mbar_wait(&sh.kv_full[h & 7], (h >> 3) & 1, &no_abort, kDrainLimitNs);
      }
    }
    __syncwarp();
  } else if (warp == 1 - prod_w) {
    // ---------------- MMA issuer (the whole warp; one elected lane issues)
    struct Item { int i, j, T, e; bool valid; };  // query tile, key tile in it, its count, non-empty ordinal
    Item q0{-1, 0, 0, 0, false}, q1{-1, 0, 0, 0, false};  // key tiles g-2 and g-1, while their PV is pending
    int g = 0, e = 0, kslot = 0, vslot = 0;
    bool ok = true;
    // PV of key tile h = g - 2 (or later in the drain).
    auto pv = [&](const Item& it, int h) -> bool {
      if (!warp_wait(&sh.p_full[h & 1], (h >> 1) & 1, abort_flag)) return false;
      if (it.j == 0 && it.e >= 1 && !warp_wait(&sh.o_empty, (it.e - 1) & 1, abort_flag)) return false;
      tc_fence_after();
      issue_pv<D>(tmem + kOCol, tmem + (h & 1) * 64, sbase + L::kOffV + vslot * T::kKVBytes, it.j > 0);
      if (++vslot == NV) vslot = 0;
      if (it.j == it.T - 1) mma_commit_w(&sh.o_full);
      return true;
    };
    for (int i = 0; ok && i < n_mine; ++i) {
      if (!warp_wait(&sh.list_full[i % NL], (i / NL) & 1, abort_flag)) { ok = false; break; }
      const int Tn = lists[(i % NL) * cap];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.list_empty[i % NL]);
      if (Tn == 0) continue;
      // Q(i) reuses the buffer that tile i-2's output is stored from, which needs every PV of
      // i-2; after a query tile with a single key tile one may still be pending: issue it now
      // (the later step commits still cover it).
      if (ok && q0.valid && q0.i <= i - 2) {
        ok = pv(q0, g - 2);
        q0.valid = false;
      }
      if (ok && q1.valid && q1.i <= i - 2) {
        ok = pv(q1, g - 1);
        q1.valid = false;
      }
      if (!ok) break;
      if (!warp_wait(&sh.q_full[i & 1], (i >> 1) & 1, abort_flag)) { ok = false; break; }
      const uint32_t q_base = sbase + L::kOffQ + (i & 1) * T::kQBytes;
      const uint32_t q_tm = tmem + kQCol + (e & 1) * 32;  // head dim 64: Q of the e-th non-empty tile
      for (int j = 0; j < Tn; ++j, ++g) {
        if (q0.valid && !pv(q0, g - 2)) { ok = false; break; }
        // P(g-2) consumed means every QK^T up to g-2 is done, in particular those of the
        // non-empty tile e-2, the last reader of this Q buffer.
        if constexpr (kQTmem) {
          if (j == 0) copy_q_to_tmem<D>(q_tm, q_base);
        }
        if (!warp_wait(&sh.kv_full[g & 7], (g >> 3) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_base = sbase + L::kOffK + kslot * T::kKVBytes;
        if constexpr (kQTmem) issue_qk_tq<D>(tmem + (g & 1) * 64, q_tm, k_base);
        else issue_qk<D>(tmem + (g & 1) * 64, q_base, k_base);
        mma_commit_w(&sh.step[g & 7]);
        if (++kslot == NK) kslot = 0;
        q0 = q1;
        q1 = Item{i, j, Tn, e, true};
      }
      ++e;
    }
    // Drain: the last two PVs, each closing a step of its own.
    if (ok && q0.valid) ok = pv(q0, g - 2);
    if (ok) mma_commit_w(&sh.step[g & 7]);
    if (ok && q1.valid) ok = pv(q1, g - 1);
    if (ok) mma_commit_w(&sh.step[(g + 1) & 7]);
    mma_commit_w(&sh.drain);
    volatile int no_abort = 0;
    mbar_wait(&sh.drain, 0, &no_abort, kDrainLimitNs);
    __syncwarp();
  } else {
    // ---------------- softmax + epilogue: one query row per thread (warps 2..5)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int grp = r / BS;
    const float C = a.scale_log2;
    const uint64_t C2 = f2_pack(C, C);
    constexpr int kUBytes = kU16 ? D * 2 : D * 4;  // one cached U row
    // Prefetch into L2 the row of U that the epilogue of tile i reads.
    auto prefetch_u = [&](int i) {
      if (!has_stats || i >= n_mine) return;
      const int t = tile_of(i), bh = t / n_qt, qb = tile_query_block<BS>(a, n_qt, bh, t % n_qt, r / BS);
      const int row = qb * BS + r % BS;
      if (qb < 0 || row >= a.N) return;
      const size_t rg = static_cast<size_t>(bh) * a.N + row;
      const unsigned char* u = kU16 ? reinterpret_cast<const unsigned char*>(a.stat_u16 + rg * D)
                                    : reinterpret_cast<const unsigned char*>(a.stat_u + rg * D);
#pragma unroll
      for (int off = 0; off < kUBytes; off += 128) prefetch_l2(u + off);
      prefetch_l2(u + kUBytes - 4);
    };
    // This row's cached m, Z_full, Z_kept (and U's scale) for tile i, read a tile ahead into
    // registers (the neutral 0, 1, 1, 1 for rows past N or without statistics).
    auto load_stats = [&](int i, float& m, float& zf, float& zk, float& us) {
      m = 0.f;
      zf = 1.f;
      zk = 1.f;
      us = 1.f;
      if (!has_stats || i >= n_mine) return;
      const int t = tile_of(i), bh = t / n_qt, qb = tile_query_block<BS>(a, n_qt, bh, t % n_qt, r / BS);
      const int row = qb * BS + r % BS;
      if (qb < 0 || row >= a.N) return;
      const size_t rg = static_cast<size_t>(bh) * a.N + row;
      m = __ldg(a.stat_m + rg);
      zf = __ldg(a.stat_zfull + rg);
      zk = __ldg(a.stat_zkept + rg);
      if constexpr (kU16) us = __ldg(a.stat_u_scale + rg);
    };
    prefetch_u(0);
    float next_m, next_zf, next_zk, next_us;
    load_stats(0, next_m, next_zf, next_zk, next_us);
    int g = 0, e = 0;
    for (int i = 0; i < n_mine; ++i) {
      prefetch_u(i + 1);
      const int t = tile_of(i), bh = t / n_qt, qt = t % n_qt;
      const int qb = tile_query_block<BS>(a, n_qt, bh, qt, r / BS);
      const int row = qb * BS + r % BS;
      const bool valid = qb >= 0 && row < a.N;
      const size_t row_g = static_cast<size_t>(bh) * a.N + (valid ? row : 0);
      const float mc2 = next_m * kLog2e, zf_c = next_zf, zk_c = next_zk, us_c = next_us;
      load_stats(i + 1, next_m, next_zf, next_zk, next_us);
      float m_run = has_stats ? mc2 : -INFINITY;
      const int lb = i % NL;
      if (!warp_wait(&sh.list_full[lb], (i / NL) & 1, abort_flag)) break;
      const int Tn = lists[lb * cap];
      const uint16_t* lst = lists + lb * cap + 1;
      float m_seen = -INFINITY, z = 0.f;
      bool ok = true;
      for (int j = 0; j < Tn; ++j, ++g) {
        const uint32_t ent = lst[j];  // the list is complete: read it while S(g) is computed
        if (!warp_wait(&sh.step[g & 7], (g >> 3) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const bool active = (ent >> grp) & 1u;  // warp-uniform
        const uint32_t pt = tmem + lane_off + (g & 1) * 64;
        uint32_t pk[32];
        if (active) {
          float s[64];
          tmem_ld64(pt, s);
          mask_tail(s, static_cast<int>(ent >> 2) * kBN, a.N);
          // With a finite reference m' (the capture step's row max, or an earlier key tile's)
          // the exponentials need no row max: only a tile sum above 2^kRescaleUp (some p may be
          // that large) or a row total below 2^-kRescaleDown (all of it negligible) sends the
          // warp to the max-based path, which recomputes the tile.
          bool slow = true;
          if (__all_sync(0xffffffffu, m_run != -INFINITY)) {
            const float zt = exp_row64(s, m_run, C2, pk);
            slow = __any_sync(0xffffffffu, !(zt <= kSumUp) || z + zt < kSumDown);
            if (!slow) z += zt;
          }
          if (slow) {
            // The earlier tiles' scores are at most m' + log2(z): none of their p exceeds z.
            if (z > 0.f) m_seen = fmaxf(m_seen, m_run + __log2f(z));
            m_seen = fmaxf(m_seen, row_max64(s) * C);
            float ref = m_run;
            bool need = false;
            if (m_run == -INFINITY) {
              ref = m_seen;
            } else if (m_seen > m_run + kRescaleUp || m_seen < m_run - kRescaleDown) {
              need = true;
              ref = m_seen;
            }
            if (__any_sync(0xffffffffu, need)) {
              // Rescaling O needs PV(g-1) done: step g+1 (the previous tile's O is already read when j == 0).
              if (j > 0 && !warp_wait(&sh.step[(g + 1) & 7], ((g + 1) >> 3) & 1, abort_flag)) { ok = false; break; }
              tc_fence_after();
              // Moving the reference down (the row so far far below the cached max) multiplies
              // by up to 2^126 while anything has been summed (a term >= 2^-126 bounds the gap);
              // with nothing summed yet O and z are zero and the factor could overflow, so 0.
              const float f = need ? (z > 0.f ? ex2_approx(m_run - ref) : 0.f) : 1.f;
              tmem_row_scale<D>(tmem + lane_off + kOCol, f);
              z *= f;
            }
            m_run = ref;
            if (m_run == -INFINITY) {
#pragma unroll
              for (int c = 0; c < 32; ++c) pk[c] = 0u;
            } else {
              z += exp_row64(s, m_run, C2, pk);
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = 0u;
        }
        tmem_st32(pt, pk);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sh.p_full[g & 1]);
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.list_empty[lb]);

      // ---- epilogue
      // U's first kUPre columns are read before waiting for O so their latency overlaps the
      // last PV, the rest as each 16-column chunk is combined.  Measured: 32 of 64 columns is
      // ~1.5% faster than all 64 (whose registers the loop then lacks), 48 of 80 ~7% faster
      // than all 80 on the long-image workload.
      constexpr int kUPre = D == 64 ? 32 : (D == 80 ? 48 : 64);
      const bool has_u = has_stats && valid;
      const float4* up = reinterpret_cast<const float4*>(a.stat_u + row_g * D);
      const uint4* up16 = reinterpret_cast<const uint4*>(a.stat_u16 + row_g * D);
      float u[kUPre];
#pragma unroll
      for (int c = 0; c < kUPre; ++c) u[c] = 0.f;
      float fu = 0.f;
      if (has_u) {
        if constexpr (kU16) {
#pragma unroll
          for (int q8 = 0; q8 < kUPre / 8; ++q8) {
            const uint4 x = __ldg(up16 + q8);
            const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) f16x2_to_f32(w4[h], u[8 * q8 + 2 * h], u[8 * q8 + 2 * h + 1]);
          }
        } else {
#pragma unroll
          for (int q4 = 0; q4 < kUPre / 4; ++q4) {
            const float4 x = __ldg(up + q4);
            u[4 * q4 + 0] = x.x;
            u[4 * q4 + 1] = x.y;
            u[4 * q4 + 2] = x.z;
            u[4 * q4 + 3] = x.w;
          }
        }
        fu = ex2_approx(mc2 - m_run) * us_c;  // us_c: U's power-of-two scale (1 for fp32 U)
      }
      const float denom = has_stats ? z * (zf_c / zk_c) : z;
      float inv = z > 0.f ? 1.f / denom : 0.f;
      // o = (N' + e^{m_c - m'} U) * inv.  On a row whose kept keys lie far below its masked
      // maximum, inv can underflow and e^{m_c - m'} U overflow although their product is of
      // the order of |v|; there inv is raised to 2^-100 (N' * inv stays negligible, as the
      // true value is smaller still) and U's coefficient is formed in the log domain with
      // 2^100 taken out.  A cached Z_kept of 0 there means a kept mass below the cache's
      // range (under ~2^-226 of the row's): the row is reshaped as if it had not changed
      // since the capture, o = U / Z_full.
      if (has_u && z > 0.f && !(inv >= 0x1p-100f && mc2 - m_run < 120.f)) {
        inv = 0x1p-100f;
        fu = far_row_u_coef(mc2 - m_run, zk_c, zf_c, z) * us_c;
      }
      unsigned char* stg = smem + L::kOffQ + (i & 1) * T::kQBytes;
      if (Tn > 0) {
        if (!warp_wait(&sh.o_full, e & 1, abort_flag)) break;
        tc_fence_after();
      } else {
        // No key tile: the Q load of this tile must land before its buffer is reused.
        if (!warp_wait(&sh.q_full[i & 1], (i >> 1) & 1, abort_flag)) break;
      }
      // O (16 columns at a time) + e^{m_c - m'} U, normalised, as bf16 into the tile's Q
      // buffer in the 128B / 32B swizzled layouts the TMA store expects.
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 16) {
        float v[16];
        if (Tn > 0) {
          tmem_ld16(tmem + lane_off + kOCol + c0, v);
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) v[c] = 0.f;
        }
        float uc[16];
        if (c0 < kUPre) {
#pragma unroll
          for (int c = 0; c < 16; ++c) uc[c] = u[(c0 < kUPre ? c0 : 0) + c];
        } else if constexpr (kU16) {
#pragma unroll
          for (int q8 = 0; q8 < 2; ++q8) {
            const uint4 x = has_u ? __ldg(up16 + c0 / 8 + q8) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) f16x2_to_f32(w4[h], uc[8 * q8 + 2 * h], uc[8 * q8 + 2 * h + 1]);
          }
        } else {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float4 x = has_u ? __ldg(up + c0 / 4 + q4) : make_float4(0.f, 0.f, 0.f, 0.f);
            uc[4 * q4 + 0] = x.x;
            uc[4 * q4 + 1] = x.y;
            uc[4 * q4 + 2] = x.z;
            uc[4 * q4 + 3] = x.w;
          }
        }
        uint32_t w[8];
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          const float v0 = (c0 + c < a.d) ? fmaf(fu, uc[c], v[c]) * inv : 0.f;
          const float v1 = (c0 + c + 1 < a.d) ? fmaf(fu, uc[c + 1], v[c + 1]) * inv : 0.f;
          w[c / 2] = pack_bf16x2(v0, v1);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c8 = c0 + 8 * h;
          unsigned char* dst;
          if (c8 < 64) dst = stg + r * 128 + (((c8 >> 3) ^ (r & 7)) << 4);
          else if (T::kTailWide) dst = stg + T::kQMain + r * 128 + ((((c8 - 64) >> 3) ^ (r & 7)) << 4);
          else dst = stg + T::kQMain + r * 32 + ((((c8 - 64) >> 3) ^ ((r >> 2) & 1)) << 4);
          *reinterpret_cast<uint4*>(dst) = make_uint4(w[4 * h], w[4 * h + 1], w[4 * h + 2], w[4 * h + 3]);
        }
      }
      if (Tn > 0) {
        tc_fence_before();
        mbar_arrive(&sh.o_empty);
        ++e;
      }
      fence_proxy_async_smem();
      mbar_arrive(&sh.staged[i & 1]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ================================================================== capture step
//
// One CTA per 128-row query tile, every key tile in order.  Each key tile's
// P V goes to O_kept (rows whose query block keeps the tile's block) and/or
// to U (the other rows).  The PV products take P in f16 with V in f16 (an f16
// copy of V made by convert_v_f16_kernel before the launch, scaled per head
// by a power of two that puts max |v| in [2^14, 2^15), undone exactly in the
// epilogue), in one product per key tile.  The kept and the masked keys of a
// row are two online softmaxes with references of their own, and P enters f16
// as p * 2^7 (p <= 2^8 under the lazy reference, so P <= 2^15): a masked term
// down to 2^-21 of the row's largest masked term keeps 11 mantissa bits (a
// rounding error below 2^-12), a smaller one an absolute error below 2^-32 of
// it, wherever the row's maximum lies.
//
// S is double-buffered in TMEM, so QK^T(j+1) runs while the softmax works on
// tile j: the MMA warp issues QK^T(j+1) as soon as PV(j-1) -- the last reader
// of that buffer -- is issued, then waits for P(j) and issues PV(j).
// A tile that is kept by some rows and masked for others ("mixed"; a few per
// cent of the tiles) needs P twice: the masked rows' P stays in the S buffer
// (kept rows zero) for the U product, and the kept rows' P goes to a
// shared-memory tile (masked rows zero) read by one SS product into O_kept.
// TMEM: S0 [0,64) S1 [64,128) O_kept [128,128+D) U at kOUCol.  Head dim 64
// fits in 256 columns, so two CTAs share an SM (two softmax warps per SM
// sub-partition); head dim 80 takes 512 columns and one CTA per SM.
template <int D>
struct CaptureLayout {
  using T = Tiles<D>;
  static constexpr uint32_t kTmemCols = D == 64 ? 256 : 512;
  static constexpr uint32_t kOKCol = 128;
  static constexpr uint32_t kOUCol = D == 64 ? 192 : 256;
  static constexpr int kStages = 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffStage0 = T::kQBytes;
  static constexpr int kOffPK = kOffStage0 + kStages * T::kStageBytes;  // 128 x 64 f16, 128-byte swizzle
  static constexpr int kOffShared = kOffPK + kBM * 128;
  static constexpr size_t kMinSmem = D == 64 ? 0 : 120 * 1024;  // D > 64: keep one CTA per SM
};

struct alignas(8) CaptureShared {
  uint64_t q_full;
  uint64_t kv_full[4], kv_empty[4];
  uint64_t s_full[2], p_full[2];
  uint64_t pk_free, o_full, drain;
  uint32_t tmem_base;
  int abort_flag;
  int ok_any;  // some tile is kept by some row
  int ou_any;  // some tile is masked for some row
};

template <int D>
__host__ __device__ constexpr size_t capture_smem_bytes(int n_blocks) {
  const size_t s = 1024 + CaptureLayout<D>::kOffShared + sizeof(CaptureShared) + 2 * sizeof(uint32_t) * attn_words(n_blocks) +
                   2 * static_cast<size_t>(n_blocks);
  return s > CaptureLayout<D>::kMinSmem ? s : CaptureLayout<D>::kMinSmem;
}

// acc (+)= P V with P (128 x 64 f16) in shared memory, K-major with 128-byte swizzle, and f16 V.
template <int D>
__device__ __forceinline__ void issue_pv_ss(uint32_t acc_tmem, uint32_t p_base, uint32_t v_base, bool accumulate) {
  const uint64_t pd = smem_desc(p_base, 16, 1024, kSwizzle128B);
  const uint64_t vd = smem_desc(v_base, Tiles<D>::kKVMain, 1024, kSwizzle128B);
  const uint32_t acc0 = accumulate ? 1u : 0u;
  mma_ss_w(acc_tmem, pd, vd, kIdescPV64F16, acc0);
#pragma unroll
  for (int ks = 1; ks < kBN / 16; ++ks) mma_ss_w(acc_tmem, pd + 2 * ks, vd + 128 * ks, kIdescPV64F16, 1u);
  if constexpr (Tiles<D>::kTail) {
    using T = Tiles<D>;
    const uint64_t vt = smem_desc(v_base + T::kKVMain, T::kKVTail, T::kTailSBO, T::kTailSwizzle);
    mma_ss_w(acc_tmem + 64, pd, vt, T::kIdescPVTailF16, acc0);
#pragma unroll
    for (int ks = 1; ks < kBN / 16; ++ks)
      mma_ss_w(acc_tmem + 64, pd + 2 * ks, vt + T::kTailRow * ks, T::kIdescPVTailF16, 1u);
  }
}

template <int D, int BS, bool kU16>
__global__ void __launch_bounds__(kAttnThreads, 2)
    full_capture_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tq_tail,
                        const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tk_tail,
                        const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tv_tail,
                        const AttnArgs a) {
  using T = Tiles<D>;
  using L = CaptureLayout<D>;
  static_assert(BS == 64 || BS == 128, "block size must be 64 or 128");
  constexpr int kQB = kBM / BS;
  constexpr int NS = L::kStages;

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sbase = smem_u32(smem);
  CaptureShared& sh = *reinterpret_cast<CaptureShared*>(smem + L::kOffShared);
  const int words = attn_words(a.n_blocks);
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(&sh + 1);
  uint8_t* kinds = reinterpret_cast<uint8_t*>(bitmaps + 2 * attn_words(a.n_blocks));  // [key tiles]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.y;
  const int q_row0 = blockIdx.x * kBM;
  const int qb0 = blockIdx.x * kQB;
  const int nqb_here = min(kQB, a.n_blocks - qb0);
  const int Tn = key_tiles(a.N);

  if (warp == 0) tmem_alloc(&sh.tmem_base, L::kTmemCols);
  if (threadIdx.x == 32) {
    mbar_init(&sh.q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sh.kv_full[s], 1);
      mbar_init(&sh.kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.s_full[b], 1);
      mbar_init(&sh.p_full[b], 128);
    }
    mbar_init(&sh.pk_free, 1);
    mbar_init(&sh.o_full, 1);
    mbar_init(&sh.drain, 1);
    sh.abort_flag = device_status_set() ? 1 : 0;  // an earlier failure: do nothing
    sh.ok_any = 0;
    sh.ou_any = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 2 * words; i += blockDim.x) bitmaps[i] = 0u;
  __syncthreads();
  const bool run = sh.abort_flag == 0;  // block-uniform
  if (run)
    for (int g = 0; g < kQB; ++g) mark_kept_blocks(bitmaps + g * words, a, bh, qb0 + g, threadIdx.x, blockDim.x);
  __syncthreads();
  if (run)
    for (int t = threadIdx.x; t < Tn; t += blockDim.x) {
      const int kb = t * kBN / BS;
      uint8_t kind = 0;
      for (int g = 0; g < nqb_here; ++g) {
        if (bitmap_has(bitmaps + g * words, kb)) {
          sh.ok_any = 1;
          kind |= static_cast<uint8_t>(1u << g);
        } else {
          sh.ou_any = 1;
        }
      }
      kinds[t] = kind;
    }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  // Two CTAs share an SM, one holding TMEM columns 0-255 and the other 256-511.  The second swaps
  // the producer and MMA roles of warps 0 and 1, so that the two MMA warps sit on different SM
  // sub-partitions (a warp's sub-partition is its index mod 4) and slow different softmax warps.
  const int prod_w = (tmem & 256u) ? 1 : 0;
  const bool ok_any = sh.ok_any != 0, ou_any = sh.ou_any != 0;
  volatile int* abort_flag = &sh.abort_flag;

  // Per key tile: does some row keep it / mask it?  From the byte written above (bit g: query
  // block g of the tile keeps it): evaluating the bitmaps here instead, once per key tile in
  // the MMA and softmax warps, cost the capture ~12%.
  const uint32_t all_kept = (1u << nqb_here) - 1u;
  auto tile_kind = [&](int j, bool& kept_any, bool& masked_any) {
    const uint32_t k = kinds[j];
    kept_any = k != 0u;
    masked_any = k != all_kept;
  };

  if (!run) {
    // an earlier kernel failed: leave the outputs untouched
  } else if (warp == prod_w) {
    if (lane == 0) {
      load_q<D>(smem + L::kOffQ, &tq, &tq_tail, &sh.q_full, q_row0, bh);
      int issued = 0;
      for (int j = 0; j < Tn; ++j) {
        const int st = j % NS;
        if (j >= NS && !mbar_wait(&sh.kv_empty[st], ((j / NS) - 1) & 1, abort_flag)) break;
        load_kv<D>(smem + L::kOffStage0 + st * T::kStageBytes, &tk, &tk_tail, &tv, &tv_tail, &sh.kv_full[st],
                   j * kBN, bh);
        issued = j + 1;
      }
      if (*abort_flag) {
        volatile int no_abort = 0;
        mbar_wait(&sh.q_full, 0, &no_abort, kDrainLimitNs);
        for (int j = issued > NS ? issued - NS : 0; j < issued; ++j)
          mbar_wait(&sh.kv_full[j % NS], (j / NS) & 1, &no_abort, kDrainLimitNs);
      }
    }
  } else if (warp == 1 - prod_w) {
    // MMA issuer: the whole warp, one elected lane issues.
    bool ok = warp_wait(&sh.q_full, 0, abort_flag);
    bool ok_started = false, ou_started = false;
    auto qk = [&](int j) -> bool {
      const int st = j % NS;
      if (!warp_wait(&sh.kv_full[st], (j / NS) & 1, abort_flag)) return false;
      tc_fence_after();
      issue_qk<D>(tmem + (j & 1) * 64, sbase + L::kOffQ, sbase + L::kOffStage0 + st * T::kStageBytes);
      mma_commit_w(&sh.s_full[j & 1]);
      return true;
    };
    auto pv = [&](int j) -> bool {
      bool kept_any, masked_any;
      tile_kind(j, kept_any, masked_any);
      if (!warp_wait(&sh.p_full[j & 1], (j >> 1) & 1, abort_flag)) return false;
      tc_fence_after();
      const uint32_t v_base = sbase + L::kOffStage0 + (j % NS) * T::kStageBytes + T::kKVBytes;
      const uint32_t sbuf = tmem + (j & 1) * 64;
      if (!masked_any) {  // kept by every row: P in the S buffer
        issue_pv<D, true>(tmem + L::kOKCol, sbuf, v_base, ok_started);
        ok_started = true;
      } else {
        issue_pv<D, true>(tmem + L::kOUCol, sbuf, v_base, ou_started);  // masked rows' P (kept rows 0)
        ou_started = true;
        if (kept_any) {  // mixed: the kept rows' P is in shared memory
          issue_pv_ss<D>(tmem + L::kOKCol, sbase + L::kOffPK, v_base, ok_started);
          ok_started = true;
          mma_commit_w(&sh.pk_free);
        }
      }
      mma_commit_w(&sh.kv_empty[j % NS]);  // K/V stage free and PV(j) done
      return true;
    };
    if (ok) ok = qk(0);
    for (int j = 0; ok && j < Tn; ++j) {
      // S[(j+1) & 1] held P(j-1), whose PV was issued in the previous iteration.
      if (j + 1 < Tn && !qk(j + 1)) { ok = false; break; }
      if (!pv(j)) { ok = false; break; }
    }
    if (ok) mma_commit_w(&sh.o_full);
    mma_commit_w(&sh.drain);
    volatile int no_abort = 0;
    mbar_wait(&sh.drain, 0, &no_abort, kDrainLimitNs);
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int grp = r / BS;
    const int i = q_row0 + r;
    const bool valid = i < a.N;
    const size_t row_g = static_cast<size_t>(bh) * a.N + (valid ? i : 0);
    const float C = a.scale_log2;
    // The kept keys (O_kept, Z_kept) and the masked keys (U, the masked sum) are two online
    // softmaxes with references of their own (log2 units): each set's p stays within 2^8 of
    // its own largest term, so the f16 P of the masked rows keeps its precision even when the
    // row's maximum sits in a kept block far above every masked score.
    float m_k = -INFINITY, m_u = -INFINITY;        // lazy references
    float seen_k = -INFINITY, seen_u = -INFINITY;  // largest score seen in each set
    float zk = 0.f, zm = 0.f;                      // sums of the biased p of each set
    bool ok = true;
    int mixed = 0;  // mixed key tiles so far
    for (int j = 0; j < Tn; ++j) {
      bool kept_any, masked_any;
      tile_kind(j, kept_any, masked_any);
      const bool kept = (kinds[j] >> grp) & 1u;  // warp-uniform (0 for a query block beyond the end)
      if (!warp_wait(&sh.s_full[j & 1], (j >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sbuf = tmem + lane_off + (j & 1) * 64;
      float s[64];
      tmem_ld64(sbuf, s);
      mask_tail(s, j * kBN, a.N);
      const float prev = kept ? m_k : m_u;
      const float seen = fmaxf(kept ? seen_k : seen_u, row_max64(s) * C);
      float ref = prev;
      bool need = false;
      if (prev == -INFINITY) ref = seen;
      else if (seen > prev + kRescaleUp) { need = true; ref = seen; }
      if (__any_sync(0xffffffffu, need)) {
        // PV(j-1) done: its commit also freed the K/V stage of tile j-1.
        if (j > 0 && !warp_wait(&sh.kv_empty[(j - 1) % NS], ((j - 1) / NS) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const float f = need ? ex2_approx(prev - ref) : 1.f;
        tmem_row_scale<D>(tmem + lane_off + (kept ? L::kOKCol : L::kOUCol), f);  // warp-uniform choice
        if (kept) zk *= f;
        else zm *= f;
      }
      if (kept) {
        m_k = ref;
        seen_k = seen;
      } else {
        m_u = ref;
        seen_u = seen;
      }
      const float m_run = ref;
      // p = 2^(s*C - m' + kPBias), two lanes of f32x2 arithmetic at a time; s now holds p.
      uint32_t pk[32];
      float zt;
      {
        const uint64_t C2 = f2_pack(C, C), nref = f2_pack(kPBias - m_run, kPBias - m_run);
        uint64_t zz = f2_pack(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          float x0, x1;
          const uint64_t xx = f2_fma(f2_pack(s[c], s[c + 1]), C2, nref);
          if (c % 16 == 14) {  // one pair in eight on the FMA pipe: the MUFU is the busier unit
            f2_unpack(f2_exp2_poly(xx), s[c], s[c + 1]);
          } else {
            f2_unpack(xx, x0, x1);
            s[c] = ex2_approx(x0);
            s[c + 1] = ex2_approx(x1);
          }
          zz = f2_add(zz, f2_pack(s[c], s[c + 1]));
          pk[c / 2] = pack_f16x2(s[c], s[c + 1]);
        }
        float z0, z1;
        f2_unpack(zz, z0, z1);
        zt = z0 + z1;
      }
      if (kept) zk += zt;
      else zm += zt;
      if (a.out_block_lse != nullptr && valid)  // coalesced: a warp's 32 rows are consecutive
        a.out_block_lse[(static_cast<size_t>(bh) * Tn + j) * a.N + i] = m_run + __log2f(zt) - kPBias;
      if (!masked_any) {
        tmem_st32(sbuf, pk);  // kept by every row
      } else {
        if (!kept) {
          tmem_st32(sbuf, pk);
        } else {
          tmem_st32_zero(sbuf);
        }
        if (kept_any) {
          // Mixed tile: the kept rows' P (masked rows zero) into the shared-memory tile, once
          // the previous mixed tile's product has read it.
          if (mixed > 0 && !warp_wait(&sh.pk_free, (mixed - 1) & 1, abort_flag)) { ok = false; break; }
          unsigned char* prow = smem + L::kOffPK + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 val = kept ? make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3])
                                   : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = val;
          }
          fence_proxy_async_smem();
          ++mixed;
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sh.p_full[j & 1]);
    }
    if (ok) ok = warp_wait(&sh.o_full, 0, abort_flag);
    tc_fence_after();
    if (ok) {
      // O and U were accumulated on V * 2^k; 2^-k (exact) takes the head's scale back out.
      const float unscale = exp2_int(-v_scale_exp(a.v_amax[bh]));
      // Refer both sets to the true row max M and take the bias out (exact powers of two
      // apart from ex2's rounding; a set with no term has reference -inf and weight 0).
      const float M = fmaxf(seen_k, seen_u);
      const float adjk = ex2_approx(m_k - kPBias - M);
      const float adju = ex2_approx(m_u - kPBias - M);
      const float zkept_m = zk * adjk, zfull_m = zkept_m + zm * adju;
      const float inv = zfull_m > 0.f ? unscale / zfull_m : 0.f;
      // Reference of the cache.  The row max M, unless the kept keys carry less than 2^-64
      // of the row's mass: relative to M their sum may then fall below fp32's range (a masked
      // key far above every kept one), so the cache takes a reference 2^sh lower, sh the
      // integer that balances the two sums' exponents (Z_kept 2^-(g+f)/2, Z_full 2^(g+f)/2 for
      // a gap of g binades and a full sum of 2^f).  The reshape formula does not depend on the
      // reference, as long as m, Z_full, Z_kept and U share it.
      int sh = 0;
      float zkept = zkept_m;
      if (zk > 0.f) {
        const float lk = __log2f(zk) + (m_k - kPBias - M);  // log2 Z_kept relative to M
        if (lk < -kCacheShiftBelow) {
          sh = min(static_cast<int>(-0.5f * (lk + __log2f(zfull_m))), kCacheShiftMax);
          zkept = ex2_approx(lk + static_cast<float>(sh));
        }
      }
      const float zfull = zfull_m * exp2_int(sh);
      float adj = adju * unscale * exp2_int(sh);
      float u_scale = 1.f;
      if constexpr (kU16) {
        // Compressed cache: the row's U as f16 times a power of two 2^-k, with k chosen so
        // that the row's largest |U| lands in [2^14, 2^15) (11 mantissa bits for every
        // element down to 2^-28 of it).  First pass: the row's largest |U|.
        float umax = 0.f;
        if (ou_any) {
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 16) {
            float ouv[16];
            tmem_ld16(tmem + lane_off + L::kOUCol + c0, ouv);
#pragma unroll
            for (int c = 0; c < 16; ++c)
              if (c0 + c < a.d) umax = fmaxf(umax, fabsf(ouv[c]));
          }
        }
        const int k = v_scale_exp(__float_as_uint(umax * adj));
        u_scale = exp2_int(-k);
        adj *= exp2_int(k);
      }
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 16) {
        float okv[16], ouv[16];
        if (ok_any) tmem_ld16(tmem + lane_off + L::kOKCol + c0, okv);
        else {
#pragma unroll
          for (int c = 0; c < 16; ++c) okv[c] = 0.f;
        }
        if (ou_any) tmem_ld16(tmem + lane_off + L::kOUCol + c0, ouv);
        else {
#pragma unroll
          for (int c = 0; c < 16; ++c) ouv[c] = 0.f;
        }
        if (valid && a.out != nullptr) {  // no O and U in the block-mass pass
          uint32_t w[8];
          float uo[16];
#pragma unroll
          for (int c = 0; c < 16; c += 2) {
            const bool in0 = c0 + c < a.d, in1 = c0 + c + 1 < a.d;
            const float o0 = in0 ? fmaf(okv[c], adjk, ouv[c] * adju) * inv : 0.f;
            const float o1 = in1 ? fmaf(okv[c + 1], adjk, ouv[c + 1] * adju) * inv : 0.f;
            w[c / 2] = pack_bf16x2(o0, o1);
            uo[c] = in0 ? ouv[c] * adj : 0.f;
            uo[c + 1] = in1 ? ouv[c + 1] * adj : 0.f;
          }
          uint4* dst = reinterpret_cast<uint4*>(a.out + row_g * D + c0);
          dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
          if constexpr (kU16) {
            uint32_t h[8];
#pragma unroll
            for (int c = 0; c < 16; c += 2) h[c / 2] = pack_f16x2(uo[c], uo[c + 1]);
            uint4* ud = reinterpret_cast<uint4*>(a.out_u16 + row_g * D + c0);
            ud[0] = make_uint4(h[0], h[1], h[2], h[3]);
            ud[1] = make_uint4(h[4], h[5], h[6], h[7]);
          } else {
            float4* ud = reinterpret_cast<float4*>(a.out_u + row_g * D + c0);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              ud[q4] = make_float4(uo[4 * q4], uo[4 * q4 + 1], uo[4 * q4 + 2], uo[4 * q4 + 3]);
          }
        }
      }
      if (valid) {  // the sums carry no V scale
        if constexpr (kU16) a.out_u_scale[row_g] = u_scale;
        a.out_m[row_g] = (M - static_cast<float>(sh)) * kLn2;
        a.out_zfull[row_g] = zfull;
        a.out_zkept[row_g] = zkept;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Evaluates f2_exp2_poly on n inputs (pairs of lanes), for the tests of that function.
__global__ void exp2_poly_selftest_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
  float ya, yb;
  f2_unpack(f2_exp2_poly(f2_pack(a, b)), ya, yb);
  y[i] = ya;
  if (i + 1 < n) y[i + 1] = yb;
}

// Per (batch, head) max |v| into amax (float bits, atomic max; zeroed before).  grid (x, B*H).
__global__ void __launch_bounds__(256) v_absmax_kernel(const uint4* __restrict__ v, size_t per_head8,
                                                       uint32_t* __restrict__ amax) {
  if (device_status_set()) return;  // an earlier kernel failed
  const uint4* vh = v + blockIdx.y * per_head8;
  float m = 0.f;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < per_head8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 x = __ldg(vh + i);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) m = fmaxf(m, fmaxf(fabsf(bf16_lo_to_f32(w[k])), fabsf(bf16_hi_to_f32(w[k]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax + blockIdx.y, __float_as_uint(m));
}

// f16 copy of V * 2^k (k per head from amax, see v_scale_exp), 8 elements per thread and
// step.  grid (x, B*H).
__global__ void __launch_bounds__(256) convert_v_f16_kernel(const uint4* __restrict__ v, uint4* __restrict__ v16,
                                                            size_t per_head8, const uint32_t* __restrict__ amax) {
  if (device_status_set()) return;  // an earlier kernel failed
  const float scale = exp2_int(v_scale_exp(amax[blockIdx.y]));
  const size_t base = blockIdx.y * per_head8;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < per_head8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 x = __ldg(v + base + i);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t h[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) h[k] = pack_f16x2(bf16_lo_to_f32(w[k]) * scale, bf16_hi_to_f32(w[k]) * scale);
    v16[base + i] = make_uint4(h[0], h[1], h[2], h[3]);
  }
}

// Failure-detection self test: wait on a barrier nothing completes.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, limit_ns);
}

}  // namespace rt
