// attention.cuh -- the two attention kernels of Re-ttention on tcgen05 tensor cores.
//
//   full_capture_kernel    full attention at a capture step; per row it also
//                          emits the statistics the later sparse steps reuse:
//                          row max m, Z_full, Z_kept and the fp32 residual
//                          numerator U of the masked-out keys (project page,
//                          mechanism highlight: "reusing the stable ratio between
//                          sparse and full softmax denominators and caching the
//                          residual contributions from masked-out tokens").
//   sparse_reshape_kernel  attention over the kept key blocks only, then the
//                          reshape o = (N' + e^{m_c - m'} U) / (Z' * Z_full / Z_kept)
//                          in the epilogue (teaser: "reshaping sparse attention
//                          with cached statistics across denoising steps").
//
// Shared design (one CTA = one 128-row query tile of one (batch, head)):
//  * warp 0 issues TMA loads (Q once, then K/V 64-key tiles into a 4-stage
//    ring), warp 1 issues tcgen05.mma, warps 2..5 own one query row per thread
//    (TMEM lane = row) for the softmax and the epilogue.
//  * S = Q K^T lands in TMEM (two 64-column buffers, so QK^T of tile j+1 runs
//    while the softmax of tile j does); the softmax writes P as bf16 back into
//    the first 32 columns of the same buffer and the PV product reads A = P
//    straight from TMEM (no shared-memory round trip).
//  * With 64-token blocks the 128-row tile holds two query blocks, each with
//    its own kept list; the kernel walks the union of both lists and a row
//    whose block does not keep a tile writes P = 0 for it.
//  * Online softmax in base 2 (x = s * scale * log2 e) with a lazy reference:
//    the O accumulator is rescaled only when the row max moves up by more than
//    8 (or down by more than 64 in the sparse step, whose reference starts at
//    the cached max), so the rescale path almost never runs.
//  * Head dim 64 uses 128-byte swizzled tiles; head dim 80 adds a 16-column
//    tail tile with 32-byte swizzle (one more K-step for QK^T, one N=16 MMA for PV).
//  * Every barrier wait is bounded (see ptx.cuh); on a timeout the block stops,
//    drains its own copies and MMAs, frees TMEM and returns.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace rt {

constexpr int kBM = 128;            // query rows per CTA (tcgen05 M)
constexpr int kBN = 64;             // keys per tile
constexpr int kStages = 4;          // K/V ring depth
constexpr int kAttnThreads = 192;   // 6 warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleUp = 8.f;    // log2 units
constexpr float kRescaleDown = 64.f; // log2 units
constexpr uint64_t kDrainLimitNs = 200000000ull;

template <int D>
struct Geom {
  static_assert(D == 64 || D == 80, "head_dim_padded must be 64 or 80");
  static constexpr bool kTail = D == 80;
  static constexpr int kQMain = kBM * 128;
  static constexpr int kQTail = kTail ? kBM * 32 : 0;
  static constexpr int kKVMain = kBN * 128;
  static constexpr int kKVTail = kTail ? kBN * 32 : 0;
  static constexpr int kStageBytes = 2 * (kKVMain + kKVTail);
  static constexpr int kQBytes = kQMain + kQTail;
  static constexpr int kKSteps = D / 16;
  // byte offsets from the 1024-aligned shared-memory base
  static constexpr int kOffQMain = 0;
  static constexpr int kOffQTail = kQMain;
  static constexpr int kOffStage0 = kQMain + kQTail;  // multiple of 1024
  static constexpr int kOffKMain = 0, kOffVMain = kKVMain, kOffKTail = 2 * kKVMain,
                       kOffVTail = 2 * kKVMain + kKVTail;
  static constexpr int kOffBarriers = kOffStage0 + kStages * kStageBytes;
};

struct AttnArgs {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  // sparse step: cached statistics (all null = plain block-sparse attention)
  const float* stat_m;
  const float* stat_zfull;
  const float* stat_zkept;
  const float* stat_u;
  // capture step: statistics out
  float* out_m;
  float* out_zfull;
  float* out_zkept;
  float* out_u;
  __nv_bfloat16* out;
  int N;
  int d;
  int n_blocks;
  float scale_log2;  // softmax scale * log2(e)
};

// Barriers and small shared state, placed after the tile buffers.
struct alignas(8) AttnShared {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done;
  uint64_t o_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int n_tiles;
  int ok_any;   // capture: some tile is kept by some row
  int ou_any;   // capture: some tile is masked for some row
};

__host__ __device__ constexpr int attn_words(int n_blocks) { return (n_blocks + 31) / 32; }

// Shared bytes: tiles + AttnShared + two block bitmaps + the tile list, plus 1 KB for alignment.
template <int D>
__host__ __device__ constexpr size_t attn_smem_bytes(int n_blocks, int n_key_tiles) {
  return 1024 + Geom<D>::kOffBarriers + sizeof(AttnShared) + 2 * sizeof(uint32_t) * attn_words(n_blocks) +
         sizeof(uint32_t) * (n_key_tiles + 1);
}

// ------------------------------------------------------------------ pieces shared by both kernels
template <int D>
__device__ __forceinline__ uint64_t q_desc(uint32_t sbase, int ks) {
  using G = Geom<D>;
  return ks < 4 ? smem_desc(sbase + G::kOffQMain + ks * 32, 16, 1024, kSwizzle128B)
                : smem_desc(sbase + G::kOffQTail, 16, 256, kSwizzle32B);
}
template <int D>
__device__ __forceinline__ uint64_t k_desc(uint32_t stage_base, int ks) {
  using G = Geom<D>;
  return ks < 4 ? smem_desc(stage_base + G::kOffKMain + ks * 32, 16, 1024, kSwizzle128B)
                : smem_desc(stage_base + G::kOffKTail, 16, 256, kSwizzle32B);
}
// V as the N-major B operand of P V: key rows are K, head-dim columns are N.
template <int D>
__device__ __forceinline__ uint64_t v_desc_main(uint32_t stage_base, int ks) {
  return smem_desc(stage_base + Geom<D>::kOffVMain + ks * 2048, Geom<D>::kKVMain, 1024, kSwizzle128B);
}
template <int D>
__device__ __forceinline__ uint64_t v_desc_tail(uint32_t stage_base, int ks) {
  return smem_desc(stage_base + Geom<D>::kOffVTail + ks * 512, Geom<D>::kKVTail, 256, kSwizzle32B);
}

constexpr uint32_t kIdescQK = idesc_bf16(kBM, kBN, false, false);
constexpr uint32_t kIdescPV64 = idesc_bf16(kBM, 64, false, true);
constexpr uint32_t kIdescPV16 = idesc_bf16(kBM, 16, false, true);

// QK^T of one key tile into the S buffer at `s_tmem`.
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint32_t sbase, uint32_t stage_base) {
#pragma unroll
  for (int ks = 0; ks < Geom<D>::kKSteps; ++ks)
    mma_ss(s_tmem, q_desc<D>(sbase, ks), k_desc<D>(stage_base, ks), kIdescQK, ks > 0 ? 1u : 0u);
}

// acc (+)= P V for one key tile; P is bf16 in TMEM at `p_tmem` (32 columns).
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t acc_tmem, uint32_t p_tmem, uint32_t stage_base, bool accumulate) {
#pragma unroll
  for (int ks = 0; ks < kBN / 16; ++ks) {
    const uint32_t acc = (accumulate || ks > 0) ? 1u : 0u;
    mma_ts(acc_tmem, p_tmem + ks * 8, v_desc_main<D>(stage_base, ks), kIdescPV64, acc);
    if constexpr (Geom<D>::kTail) mma_ts(acc_tmem + 64, p_tmem + ks * 8, v_desc_tail<D>(stage_base, ks), kIdescPV16, acc);
  }
}

// Producer: Q once, then the K/V tiles listed in `tiles` (entry >> 2 = key-tile index).
template <int D>
__device__ void produce(AttnShared& sh, unsigned char* smem, const CUtensorMap* tq, const CUtensorMap* tq_tail,
                        const CUtensorMap* tk, const CUtensorMap* tk_tail, const CUtensorMap* tv,
                        const CUtensorMap* tv_tail, const uint32_t* tiles, int n_tiles, int q_row0, int bh,
                        bool all_tiles) {
  using G = Geom<D>;
  volatile int* abort_flag = &sh.abort_flag;
  mbar_arrive_expect_tx(&sh.q_full, G::kQBytes);
  tma_load_3d(smem + G::kOffQMain, tq, &sh.q_full, 0, q_row0, bh);
  if constexpr (G::kTail) tma_load_3d(smem + G::kOffQTail, tq_tail, &sh.q_full, 64, q_row0, bh);
  int issued = 0;
  for (int j = 0; j < n_tiles; ++j) {
    const int st = j % kStages;
    if (j >= kStages && !mbar_wait(&sh.kv_empty[st], ((j / kStages) - 1) & 1, abort_flag)) break;
    const int tile = all_tiles ? j : static_cast<int>(tiles[j] >> 2);
    const int key_row0 = tile * kBN;
    unsigned char* stage = smem + G::kOffStage0 + st * G::kStageBytes;
    mbar_arrive_expect_tx(&sh.kv_full[st], G::kStageBytes);
    tma_load_3d(stage + G::kOffKMain, tk, &sh.kv_full[st], 0, key_row0, bh);
    tma_load_3d(stage + G::kOffVMain, tv, &sh.kv_full[st], 0, key_row0, bh);
    if constexpr (G::kTail) {
      tma_load_3d(stage + G::kOffKTail, tk_tail, &sh.kv_full[st], 64, key_row0, bh);
      tma_load_3d(stage + G::kOffVTail, tv_tail, &sh.kv_full[st], 64, key_row0, bh);
    }
    issued = j + 1;
  }
  if (*abort_flag) {
    // Let every copy this block started land before the block exits.
    volatile int no_abort = 0;
    mbar_wait(&sh.q_full, 0, &no_abort, kDrainLimitNs);
    for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
      mbar_wait(&sh.kv_full[j % kStages], (j / kStages) & 1, &no_abort, kDrainLimitNs);
  }
}

// Rescale `ncols` fp32 columns of this thread's TMEM row by f (warp-collective).
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

// Mask key columns at or beyond N (only the ragged last tile has any).
__device__ __forceinline__ void mask_tail(float (&s)[64], int key0, int N) {
  if (key0 + kBN > N) {
#pragma unroll
    for (int c = 0; c < 64; ++c)
      if (key0 + c >= N) s[c] = -INFINITY;
  }
}

__device__ __forceinline__ float row_max64(const float (&s)[64]) {
  float m0 = s[0], m1 = s[1], m2 = s[2], m3 = s[3];
#pragma unroll
  for (int c = 4; c < 64; c += 4) {
    m0 = fmaxf(m0, s[c]);
    m1 = fmaxf(m1, s[c + 1]);
    m2 = fmaxf(m2, s[c + 2]);
    m3 = fmaxf(m3, s[c + 3]);
  }
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

// p = 2^(s*C - ref) for 64 columns, packed as bf16 pairs; returns the fp32 sum of p.
__device__ __forceinline__ float exp_pack64(const float (&s)[64], float C, float ref, uint32_t (&pk)[32]) {
  float z0 = 0.f, z1 = 0.f;
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    const float p0 = ex2_approx(fmaf(s[c], C, -ref));
    const float p1 = ex2_approx(fmaf(s[c + 1], C, -ref));
    z0 += p0;
    z1 += p1;
    pk[c / 2] = pack_bf16x2(p0, p1);
  }
  return z0 + z1;
}

// p = 2^(s*C - ref) in place for 64 columns; returns the fp32 sum of p.
__device__ __forceinline__ float exp_inplace64(float (&s)[64], float C, float ref) {
  float z0 = 0.f, z1 = 0.f;
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    s[c] = ex2_approx(fmaf(s[c], C, -ref));
    s[c + 1] = ex2_approx(fmaf(s[c + 1], C, -ref));
    z0 += s[c];
    z1 += s[c + 1];
  }
  return z0 + z1;
}

// Block bitmaps of the kept key blocks of the (up to two) query blocks of this CTA.
__device__ __forceinline__ void load_block_bitmaps(uint32_t* bitmaps, int words, const AttnArgs& a, int bh,
                                                   int qb0, int nqb) {
  for (int g = 0; g < nqb; ++g) {
    const int qb = qb0 + g;
    if (qb >= a.n_blocks) break;
    const size_t r = static_cast<size_t>(bh) * a.n_blocks + qb;
    const int s = a.row_ptr[r], e = a.row_ptr[r + 1];
    const int len = max(0, min(e - s, a.n_blocks));
    for (int i = threadIdx.x; i < len; i += blockDim.x) {
      const int kb = a.col_idx[s + i];
      if (kb >= 0 && kb < a.n_blocks) atomicOr(&bitmaps[g * words + kb / 32], 1u << (kb % 32));
    }
  }
}

__device__ __forceinline__ bool bitmap_has(const uint32_t* bm, int kb) { return (bm[kb / 32] >> (kb % 32)) & 1u; }

// ------------------------------------------------------------------ sparse step
template <int D, int BS>
__global__ void __launch_bounds__(kAttnThreads, 2)
    sparse_reshape_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tq_tail,
                          const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tk_tail,
                          const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tv_tail,
                          const AttnArgs a) {
  using G = Geom<D>;
  static_assert(BS == 64 || BS == 128, "block size must be 64 or 128");
  constexpr int kQBPerCta = kBM / BS;
  constexpr uint32_t kTmemCols = 256;  // S0 [0,64) S1 [64,128) O [128,128+D)
  constexpr uint32_t kOCol = 128;

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sbase = smem_u32(smem);
  AttnShared& sh = *reinterpret_cast<AttnShared*>(smem + G::kOffBarriers);
  const int words = attn_words(a.n_blocks);
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(&sh + 1);
  uint32_t* tiles = bitmaps + 2 * words;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.y;
  const int q_row0 = blockIdx.x * kBM;
  const int qb0 = blockIdx.x * kQBPerCta;

  if (warp == 0) tmem_alloc(&sh.tmem_base, kTmemCols);
  if (threadIdx.x == 32) {
    mbar_init(&sh.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.kv_full[s], 1);
      mbar_init(&sh.kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.s_full[b], 1);
      mbar_init(&sh.p_full[b], 128);
    }
    mbar_init(&sh.pv_done, 1);
    mbar_init(&sh.o_full, 1);
    mbar_init(&sh.drain, 1);
    sh.abort_flag = device_status_set() ? 1 : 0;  // an earlier failure: do nothing
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 2 * words; i += blockDim.x) bitmaps[i] = 0u;
  __syncthreads();
  const bool run = sh.abort_flag == 0;  // block-uniform
  if (run) load_block_bitmaps(bitmaps, words, a, bh, qb0, kQBPerCta);
  __syncthreads();
  // Union of the kept lists as 64-key tiles: entry = tile << 2 | (kept by block 0) | (kept by block 1) << 1.
  if (warp == 2) {
    int count = 0;
    const int n_key_tiles = (a.N + kBN - 1) / kBN;
    for (int t0 = 0; t0 < n_key_tiles; t0 += 32) {
      const int tile = t0 + lane;
      uint32_t flags = 0u;
      if (tile < n_key_tiles) {
        const int kb = tile * kBN / BS;
        flags = bitmap_has(bitmaps, kb) ? 1u : 0u;
        if (kQBPerCta == 2) flags |= bitmap_has(bitmaps + words, kb) ? 2u : 0u;
      }
      const uint32_t mask = __ballot_sync(0xffffffffu, flags != 0u);
      if (flags) tiles[count + __popc(mask & ((1u << lane) - 1u))] = (static_cast<uint32_t>(tile) << 2) | flags;
      count += __popc(mask);
    }
    if (lane == 0) sh.n_tiles = count;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const int T = sh.n_tiles;
  volatile int* abort_flag = &sh.abort_flag;

  if (!run) {
    // an earlier kernel failed: leave the outputs untouched
  } else if (warp == 0) {
    if (lane == 0 && T > 0) produce<D>(sh, smem, &tq, &tq_tail, &tk, &tk_tail, &tv, &tv_tail, tiles, T, q_row0, bh, false);
  } else if (warp == 1) {
    if (lane == 0 && T > 0) {
      bool ok = mbar_wait(&sh.q_full, 0, abort_flag);
      auto pv = [&](int i) -> bool {
        if (!mbar_wait(&sh.p_full[i & 1], (i >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        issue_pv<D>(tmem + kOCol, tmem + (i & 1) * 64, sbase + G::kOffStage0 + (i % kStages) * G::kStageBytes, i > 0);
        mma_commit(&sh.kv_empty[i % kStages]);
        mma_commit(&sh.pv_done);
        return true;
      };
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % kStages;
        if (!mbar_wait(&sh.kv_full[st], (j / kStages) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        issue_qk<D>(tmem + (j & 1) * 64, sbase, sbase + G::kOffStage0 + st * G::kStageBytes);
        mma_commit(&sh.s_full[j & 1]);
        if (j > 0 && !pv(j - 1)) ok = false;
      }
      if (ok && pv(T - 1)) mma_commit(&sh.o_full);
      mma_commit(&sh.drain);
      volatile int no_abort = 0;
      mbar_wait(&sh.drain, 0, &no_abort, kDrainLimitNs);
    }
  } else {
    // ---- softmax + epilogue: one query row per thread
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int g = r / BS;
    const int i = q_row0 + r;
    const bool valid = i < a.N;
    const size_t row_g = static_cast<size_t>(bh) * a.N + (valid ? i : 0);
    const bool has_stats = a.stat_m != nullptr;
    const float C = a.scale_log2;
    float m_run = -INFINITY, mc2 = 0.f, zf_c = 1.f, zk_c = 1.f;
    if (has_stats) {
      if (valid) {
        mc2 = a.stat_m[row_g] * kLog2e;
        zf_c = a.stat_zfull[row_g];
        zk_c = a.stat_zkept[row_g];
      }
      m_run = mc2;
    }
    float m_seen = -INFINITY, z = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      if (!mbar_wait(&sh.s_full[j & 1], (j >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t e = tiles[j];
      const bool active = (e >> g) & 1u;
      const uint32_t pt = tmem + lane_off + (j & 1) * 64;
      if (active) {
        float s[64];
        tmem_ld64(pt, s);
        mask_tail(s, static_cast<int>(e >> 2) * kBN, a.N);
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
          if (j > 0 && !mbar_wait(&sh.pv_done, (j - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const float f = need ? ex2_approx(m_run - ref) : 1.f;
          tmem_row_scale<D>(tmem + lane_off + kOCol, f);
          z *= f;
        }
        m_run = ref;
        uint32_t pk[32];
        if (m_run == -INFINITY) {
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = 0u;
        } else {
          z += exp_pack64(s, C, m_run, pk);
        }
        tmem_st16(pt, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
        tmem_st16(pt + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
      } else {
        tmem_st32_zero(pt);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sh.p_full[j & 1]);
    }
    if (ok && T > 0) ok = mbar_wait(&sh.o_full, 0, abort_flag);
    tc_fence_after();
    if (ok) {
      const float fu = has_stats ? ex2_approx(mc2 - m_run) : 0.f;
      const float denom = has_stats ? z * (zf_c / zk_c) : z;
      const float inv = z > 0.f ? 1.f / denom : 0.f;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 16) {
        float o[16];
        if (T > 0) {
          tmem_ld16(tmem + lane_off + kOCol + c0, o);
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) o[c] = 0.f;
        }
        if (valid) {
          if (has_stats) {
            const float4* up = reinterpret_cast<const float4*>(a.stat_u + row_g * D + c0);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const float4 u = __ldg(up + q4);
              o[4 * q4 + 0] = fmaf(fu, u.x, o[4 * q4 + 0]);
              o[4 * q4 + 1] = fmaf(fu, u.y, o[4 * q4 + 1]);
              o[4 * q4 + 2] = fmaf(fu, u.z, o[4 * q4 + 2]);
              o[4 * q4 + 3] = fmaf(fu, u.w, o[4 * q4 + 3]);
            }
          }
          uint32_t w[8];
#pragma unroll
          for (int c = 0; c < 16; c += 2) {
            const float v0 = (c0 + c < a.d && z > 0.f) ? o[c] * inv : 0.f;
            const float v1 = (c0 + c + 1 < a.d && z > 0.f) ? o[c + 1] * inv : 0.f;
            w[c / 2] = pack_bf16x2(v0, v1);
          }
          uint4* dst = reinterpret_cast<uint4*>(a.out + row_g * D + c0);
          dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
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

// ------------------------------------------------------------------ capture step
template <int D, int BS>
__global__ void __launch_bounds__(kAttnThreads, 1)
    full_capture_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tq_tail,
                        const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tk_tail,
                        const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tv_tail,
                        const AttnArgs a) {
  using G = Geom<D>;
  static_assert(BS == 64 || BS == 128, "block size must be 64 or 128");
  constexpr int kQBPerCta = kBM / BS;
  // S0 [0,64) S1 [64,128) PK0 [128,160) PK1 [160,192) O_kept [256,256+D) U [384,384+D)
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kPKCol = 128, kOKCol = 256, kOUCol = 384;

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sbase = smem_u32(smem);
  AttnShared& sh = *reinterpret_cast<AttnShared*>(smem + G::kOffBarriers);
  const int words = attn_words(a.n_blocks);
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(&sh + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.y;
  const int q_row0 = blockIdx.x * kBM;
  const int qb0 = blockIdx.x * kQBPerCta;
  const int nqb_here = min(kQBPerCta, a.n_blocks - qb0);
  const int T = (a.N + kBN - 1) / kBN;

  if (warp == 0) tmem_alloc(&sh.tmem_base, kTmemCols);
  if (threadIdx.x == 32) {
    mbar_init(&sh.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.kv_full[s], 1);
      mbar_init(&sh.kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.s_full[b], 1);
      mbar_init(&sh.p_full[b], 128);
    }
    mbar_init(&sh.pv_done, 1);
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
  if (run) load_block_bitmaps(bitmaps, words, a, bh, qb0, kQBPerCta);
  __syncthreads();
  // Which accumulators this CTA will touch at all.
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    const int kb = t * kBN / BS;
    for (int g = 0; g < nqb_here; ++g) {
      if (bitmap_has(bitmaps + g * words, kb)) sh.ok_any = 1;
      else sh.ou_any = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const bool ok_any = sh.ok_any != 0, ou_any = sh.ou_any != 0;
  volatile int* abort_flag = &sh.abort_flag;

  // Per key tile: does some row keep it / mask it?
  auto tile_kind = [&](int j, bool& kept_any, bool& masked_any) {
    const int kb = j * kBN / BS;
    kept_any = false;
    masked_any = false;
    for (int g = 0; g < nqb_here; ++g) {
      if (bitmap_has(bitmaps + g * words, kb)) kept_any = true;
      else masked_any = true;
    }
  };

  if (!run) {
    // an earlier kernel failed: leave the outputs untouched
  } else if (warp == 0) {
    if (lane == 0) produce<D>(sh, smem, &tq, &tq_tail, &tk, &tk_tail, &tv, &tv_tail, nullptr, T, q_row0, bh, true);
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(&sh.q_full, 0, abort_flag);
      bool ok_started = false, ou_started = false;
      auto pv = [&](int i) -> bool {
        if (!mbar_wait(&sh.p_full[i & 1], (i >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        bool kept_any, masked_any;
        tile_kind(i, kept_any, masked_any);
        const uint32_t stage_base = sbase + G::kOffStage0 + (i % kStages) * G::kStageBytes;
        if (kept_any) {
          issue_pv<D>(tmem + kOKCol, tmem + kPKCol + (i & 1) * 32, stage_base, ok_started);
          ok_started = true;
        }
        if (masked_any) {
          const uint32_t sbuf = tmem + (i & 1) * 64;
          issue_pv<D>(tmem + kOUCol, sbuf, stage_base, ou_started);        // bf16(p)
          issue_pv<D>(tmem + kOUCol, sbuf + 32, stage_base, true);         // p - bf16(p)
          ou_started = true;
        }
        mma_commit(&sh.kv_empty[i % kStages]);
        mma_commit(&sh.pv_done);
        return true;
      };
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % kStages;
        if (!mbar_wait(&sh.kv_full[st], (j / kStages) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        issue_qk<D>(tmem + (j & 1) * 64, sbase, sbase + G::kOffStage0 + st * G::kStageBytes);
        mma_commit(&sh.s_full[j & 1]);
        if (j > 0 && !pv(j - 1)) ok = false;
      }
      if (ok && pv(T - 1)) mma_commit(&sh.o_full);
      mma_commit(&sh.drain);
      volatile int no_abort = 0;
      mbar_wait(&sh.drain, 0, &no_abort, kDrainLimitNs);
    }
  } else {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int g = r / BS;
    const int i = q_row0 + r;
    const bool valid = i < a.N;
    const size_t row_g = static_cast<size_t>(bh) * a.N + (valid ? i : 0);
    const float C = a.scale_log2;
    const uint32_t* my_bm = bitmaps + (g < nqb_here ? g : 0) * words;
    float m_run = -INFINITY, m_seen = -INFINITY, zk = 0.f, zm = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      if (!mbar_wait(&sh.s_full[j & 1], (j >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      bool kept_any, masked_any;
      tile_kind(j, kept_any, masked_any);
      const bool kept = g < nqb_here && bitmap_has(my_bm, j * kBN / BS);
      const uint32_t sbuf = tmem + lane_off + (j & 1) * 64;
      float s[64];
      tmem_ld64(sbuf, s);
      mask_tail(s, j * kBN, a.N);
      m_seen = fmaxf(m_seen, row_max64(s) * C);
      float ref = m_run;
      bool need = false;
      if (m_run == -INFINITY) ref = m_seen;
      else if (m_seen > m_run + kRescaleUp) { need = true; ref = m_seen; }
      if (__any_sync(0xffffffffu, need)) {
        if (j > 0 && !mbar_wait(&sh.pv_done, (j - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const float f = need ? ex2_approx(m_run - ref) : 1.f;
        tmem_row_scale<D>(tmem + lane_off + kOKCol, f);
        tmem_row_scale<D>(tmem + lane_off + kOUCol, f);
        zk *= f;
        zm *= f;
      }
      m_run = ref;
      const float zt = exp_inplace64(s, C, m_run);  // s now holds p
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) pk[c / 2] = pack_bf16x2(s[c], s[c + 1]);
      if (kept) zk += zt; else zm += zt;
      if (kept_any) {
        if (kept) {
          tmem_st16(tmem + lane_off + kPKCol + (j & 1) * 32, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
          tmem_st16(tmem + lane_off + kPKCol + (j & 1) * 32 + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
        } else {
          tmem_st32_zero(tmem + lane_off + kPKCol + (j & 1) * 32);
        }
      }
      if (masked_any) {
        if (!kept) {
          uint32_t lo[32];  // residual p - bf16(p), so U keeps ~16 mantissa bits of p
#pragma unroll
          for (int c = 0; c < 64; c += 2)
            lo[c / 2] = pack_bf16x2(s[c] - bf16_lo_to_f32(pk[c / 2]), s[c + 1] - bf16_hi_to_f32(pk[c / 2]));
          tmem_st16(sbuf, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
          tmem_st16(sbuf + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
          tmem_st16(sbuf + 32, *reinterpret_cast<const uint32_t(*)[16]>(&lo[0]));
          tmem_st16(sbuf + 48, *reinterpret_cast<const uint32_t(*)[16]>(&lo[16]));
        } else {
          tmem_st32_zero(sbuf);
          tmem_st32_zero(sbuf + 32);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sh.p_full[j & 1]);
    }
    if (ok) ok = mbar_wait(&sh.o_full, 0, abort_flag);
    tc_fence_after();
    if (ok) {
      const float adj = ex2_approx(m_run - m_seen);  // <= 1: refer the cache to the true row max
      const float zsum = zk + zm;
      const float inv = zsum > 0.f ? 1.f / zsum : 0.f;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 16) {
        float okv[16], ouv[16];
        if (ok_any) tmem_ld16(tmem + lane_off + kOKCol + c0, okv);
        else {
#pragma unroll
          for (int c = 0; c < 16; ++c) okv[c] = 0.f;
        }
        if (ou_any) tmem_ld16(tmem + lane_off + kOUCol + c0, ouv);
        else {
#pragma unroll
          for (int c = 0; c < 16; ++c) ouv[c] = 0.f;
        }
        if (valid) {
          uint32_t w[8];
          float uo[16];
#pragma unroll
          for (int c = 0; c < 16; c += 2) {
            const bool in0 = c0 + c < a.d, in1 = c0 + c + 1 < a.d;
            const float o0 = in0 ? (okv[c] + ouv[c]) * inv : 0.f;
            const float o1 = in1 ? (okv[c + 1] + ouv[c + 1]) * inv : 0.f;
            w[c / 2] = pack_bf16x2(o0, o1);
            uo[c] = in0 ? ouv[c] * adj : 0.f;
            uo[c + 1] = in1 ? ouv[c + 1] * adj : 0.f;
          }
          uint4* dst = reinterpret_cast<uint4*>(a.out + row_g * D + c0);
          dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
          float4* ud = reinterpret_cast<float4*>(a.out_u + row_g * D + c0);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) ud[q4] = make_float4(uo[4 * q4], uo[4 * q4 + 1], uo[4 * q4 + 2], uo[4 * q4 + 3]);
        }
      }
      if (valid) {
        a.out_m[row_g] = m_seen * kLn2;
        a.out_zfull[row_g] = (zk + zm) * adj;
        a.out_zkept[row_g] = zk * adj;
      }
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
