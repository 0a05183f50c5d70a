// rettention.cu -- host side of the C ABI declared in include/rettention.h.
//
// Validates every argument before touching CUDA, encodes the TMA tensor maps,
// and launches the kernels of mask_builder.cuh and attention.cuh on the
// caller's stream.  All kernels live in this one translation unit so that the
// device status word is a single symbol of one module.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "rettention.h"
#include "ptx.cuh"
#include "mask_builder.cuh"
#include "attention.cuh"
#include "pairing.cuh"
#include "hilbert.cuh"

namespace {

using rt::AttnArgs;

constexpr int kMaxBlocks = 2048;
// The sparse kernel's producer keeps two query blocks' kept-block bitmaps in shared memory.
static_assert(2 * rt::attn_words(kMaxBlocks) <= 2 * 64, "sparse list scratch too small");

// ------------------------------------------------------------------ validation
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Dims {
  int64_t B, H, N, d, D, bs, n_blocks, bh;
};

rt_status check_shape(const rt_shape* s, Dims* out) {
  if (s == nullptr) return RT_ERR_INVALID_ARGUMENT;
  if (s->batch <= 0 || s->heads <= 0 || s->seq_len <= 0 || s->head_dim <= 0 || s->head_dim_padded <= 0 ||
      s->block_size <= 0)
    return RT_ERR_INVALID_ARGUMENT;
  if (s->head_dim > s->head_dim_padded) return RT_ERR_INVALID_ARGUMENT;
  if (s->head_dim_padded != 64 && s->head_dim_padded != 80 && s->head_dim_padded != 128) return RT_ERR_UNSUPPORTED;
  if (s->block_size != 64 && s->block_size != 128) return RT_ERR_UNSUPPORTED;
  Dims d;
  d.B = s->batch;
  d.H = s->heads;
  d.N = s->seq_len;
  d.d = s->head_dim;
  d.D = s->head_dim_padded;
  d.bs = s->block_size;
  d.n_blocks = (d.N + d.bs - 1) / d.bs;
  d.bh = d.B * d.H;
  if (d.n_blocks > kMaxBlocks) return RT_ERR_UNSUPPORTED;
  if (d.bh > 65535) return RT_ERR_UNSUPPORTED;                 // grid.y
  if (d.bh * d.N > (int64_t(1) << 31) - 1) return RT_ERR_UNSUPPORTED;  // row ids stay in int32 range
  *out = d;
  return RT_OK;
}

bool scale_ok(float scale) { return std::isfinite(scale) && scale > 0.f; }

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 (or f16) tensor [bh][N][D] viewed as 3-D (D, N, bh); box of `box_cols` x `box_rows` x 1.
bool make_map(CUtensorMap* m, const void* base, const Dims& d, int box_cols, int box_rows, bool swizzle128,
              CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d.D), static_cast<cuuint64_t>(d.N), static_cast<cuuint64_t>(d.bh)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d.D * 2), static_cast<cuuint64_t>(d.N * d.D * 2)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, type, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct Maps {
  CUtensorMap q, q_tail, k, k_tail, v, v_tail, o, o_tail;
};

// Q and O boxes are `q_rows` high: a whole 128-row tile for the capture kernel, one
// query block for the sparse kernel (whose tiles may pair any two blocks of a head).
// V is f16 for the capture kernel (v_f16), bf16 otherwise.
bool make_maps(Maps* m, const Dims& d, const void* q, const void* k, const void* v, const void* out, int q_rows,
               bool v_f16 = false) {
  std::memset(m, 0, sizeof(*m));
  const CUtensorMapDataType vt = v_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  bool ok = make_map(&m->q, q, d, 64, q_rows, true) && make_map(&m->k, k, d, 64, rt::kBN, true) &&
            make_map(&m->v, v, d, 64, rt::kBN, true, vt) && make_map(&m->o, out, d, 64, q_rows, true);
  if (d.D > 64) {
    // Columns 64..D-1: 16 of them (32-byte swizzle) for D = 80, 64 (128-byte swizzle) for D = 128.
    const int tc = static_cast<int>(d.D) - 64;
    const bool wide = tc == 64;
    ok = ok && make_map(&m->q_tail, q, d, tc, q_rows, wide) && make_map(&m->k_tail, k, d, tc, rt::kBN, wide) &&
         make_map(&m->v_tail, v, d, tc, rt::kBN, wide, vt) && make_map(&m->o_tail, out, d, tc, q_rows, wide);
  } else {
    m->q_tail = m->q;
    m->k_tail = m->k;
    m->v_tail = m->v;
    m->o_tail = m->o;
  }
  return ok;
}

int sm_count() {
  static int counts[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (counts[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    counts[dev] = n;
  }
  return counts[dev];
}

rt_status launch_status() { return cudaGetLastError() == cudaSuccess ? RT_OK : RT_ERR_CUDA; }

// The mask builder's transient workspace (pooled block means) comes from a
// stream-ordered memory pool owned by the library, one per device, that keeps
// freed memory cached instead of returning it to the driver at every
// synchronisation: repeated calls then never wait in the driver's allocator.
cudaMemPool_t workspace_pool() {
  static std::mutex mu;
  static cudaMemPool_t pools[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (pools[dev] == nullptr) {
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
    uint64_t keep = ~0ull;
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    pools[dev] = pool;
  }
  return pools[dev];
}

bool workspace_alloc(void** p, size_t bytes, cudaStream_t s) {
  cudaMemPool_t pool = workspace_pool();
  if (pool == nullptr) return false;
  return cudaMallocFromPoolAsync(p, bytes, pool, s) == cudaSuccess;
}

// ------------------------------------------------------------------ attention launch
// Shared-memory size and the largest carveout, so two CTAs fit on an SM when their sizes allow.
template <typename K>
bool set_smem(K kernel, size_t smem) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) ==
             cudaSuccess &&
         cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                              static_cast<int>(cudaSharedmemCarveoutMaxShared)) == cudaSuccess;
}

template <int D, int BS, bool kU16>
rt_status launch_sparse(const Dims& d, const Maps& m, const AttnArgs& a, cudaStream_t stream) {
  // One persistent kernel; it builds each query tile's key-tile list from the CSR itself.
  const int N = static_cast<int>(d.N);
  const int64_t tiles = rt::query_tiles(N) * d.bh;
  const size_t smem = rt::sparse_smem_bytes<D>(N);
  auto kernel = rt::sparse_reshape_kernel<D, BS, kU16>;
  if (!set_smem(kernel, smem)) return RT_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(tiles, 2 * sm_count()));
  kernel<<<grid, rt::kAttnThreads, smem, stream>>>(m.q, m.q_tail, m.k, m.k_tail, m.v, m.v_tail, m.o, m.o_tail, a);
  return launch_status();
}

template <int D, int BS, bool kU16>
rt_status launch_capture(const Dims& d, const Maps& m, const AttnArgs& a, cudaStream_t stream) {
  const size_t smem = rt::capture_smem_bytes<D>(static_cast<int>(d.n_blocks));
  auto kernel = rt::full_capture_kernel<D, BS, kU16>;
  if (!set_smem(kernel, smem)) return RT_ERR_CUDA;
  dim3 grid(static_cast<unsigned>(rt::query_tiles(static_cast<int>(d.N))), static_cast<unsigned>(d.bh));
  kernel<<<grid, rt::kAttnThreads, smem, stream>>>(m.q, m.q_tail, m.k, m.k_tail, m.v, m.v_tail, a);
  return launch_status();
}

template <bool kCapture, bool kU16>
rt_status dispatch_attention_u(const Dims& d, const Maps& m, const AttnArgs& a, cudaStream_t s) {
  if (kCapture) {
    if (d.D == 64 && d.bs == 64) return launch_capture<64, 64, kU16>(d, m, a, s);
    if (d.D == 64 && d.bs == 128) return launch_capture<64, 128, kU16>(d, m, a, s);
    if (d.D == 80 && d.bs == 64) return launch_capture<80, 64, kU16>(d, m, a, s);
    if (d.D == 80 && d.bs == 128) return launch_capture<80, 128, kU16>(d, m, a, s);
    if (d.D == 128 && d.bs == 64) return launch_capture<128, 64, kU16>(d, m, a, s);
    if (d.D == 128 && d.bs == 128) return launch_capture<128, 128, kU16>(d, m, a, s);
  } else {
    if (d.D == 64 && d.bs == 64) return launch_sparse<64, 64, kU16>(d, m, a, s);
    if (d.D == 64 && d.bs == 128) return launch_sparse<64, 128, kU16>(d, m, a, s);
    if (d.D == 80 && d.bs == 64) return launch_sparse<80, 64, kU16>(d, m, a, s);
    if (d.D == 80 && d.bs == 128) return launch_sparse<80, 128, kU16>(d, m, a, s);
    if (d.D == 128 && d.bs == 64) return launch_sparse<128, 64, kU16>(d, m, a, s);
    if (d.D == 128 && d.bs == 128) return launch_sparse<128, 128, kU16>(d, m, a, s);
  }
  return RT_ERR_UNSUPPORTED;
}

// kU16: the residual numerator U is cached as f16 with a per-row power-of-two scale.
template <bool kCapture>
rt_status dispatch_attention(const Dims& d, const Maps& m, const AttnArgs& a, bool u16, cudaStream_t s) {
  return u16 ? dispatch_attention_u<kCapture, true>(d, m, a, s) : dispatch_attention_u<kCapture, false>(d, m, a, s);
}

// ------------------------------------------------------------------ mask launch
template <int D>
rt_status launch_mask(const Dims& d, const void* q, const void* k, float scale, int keep, int forced,
                      int32_t* row_ptr, int32_t* col_idx, float* scores, float* pooled, cudaStream_t stream) {
  float* pq = pooled;
  float* pk = pooled + d.bh * d.n_blocks * D;
  constexpr int kPoolThreads = D / 8 * rt::kPoolRowGroups;
  dim3 pgrid(static_cast<unsigned>(d.n_blocks), static_cast<unsigned>(d.bh), 2);
  rt::pool_blocks_kernel<D><<<pgrid, kPoolThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), static_cast<int>(d.N),
      static_cast<int>(d.d), static_cast<int>(d.bs), pq, pk);
  if (launch_status() != RT_OK) return RT_ERR_CUDA;
  const size_t smem = rt::score_select_smem_bytes<D>(static_cast<int>(d.n_blocks));
  if (cudaFuncSetAttribute(rt::score_select_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return RT_ERR_CUDA;
  dim3 sgrid(static_cast<unsigned>((d.n_blocks + rt::kSelWarps - 1) / rt::kSelWarps), static_cast<unsigned>(d.bh));
  rt::score_select_kernel<D><<<sgrid, 32 * rt::kSelWarps, smem, stream>>>(
      pq, pk, static_cast<int>(d.n_blocks), static_cast<int>(d.bs), scale, keep, forced, row_ptr, col_idx, scores);
  return launch_status();
}

// Fixed workspace of rt_build_block_mask_static: pooled Q and K means.  It is
// placed in device memory when the module loads on a device, so the call that
// uses it never allocates.
constexpr size_t kStaticPoolFloats = size_t(2) * 1024 * 1024;  // 8 MiB
static __device__ __align__(256) float g_static_pool[kStaticPoolFloats];

rt_status mask_for_dim(const Dims& d, const void* q, const void* k, float scale, int keep, int forced,
                       int32_t* row_ptr, int32_t* col_idx, float* block_scores, float* pooled, cudaStream_t s) {
  if (d.D == 64) return launch_mask<64>(d, q, k, scale, keep, forced, row_ptr, col_idx, block_scores, pooled, s);
  if (d.D == 80) return launch_mask<80>(d, q, k, scale, keep, forced, row_ptr, col_idx, block_scores, pooled, s);
  return launch_mask<128>(d, q, k, scale, keep, forced, row_ptr, col_idx, block_scores, pooled, s);
}

constexpr int kMaxDevices = 64;
std::mutex g_static_pool_mutex;
struct StaticPoolEntry {
  unsigned long long ctx_id;  // the CUDA context the address belongs to (0: none yet)
  float* addr;
};
StaticPoolEntry g_static_pool_addr[kMaxDevices] = {};

// Unique id of the calling thread's current CUDA context (0 if there is none or the driver
// cannot say).  Context ids are never reused within a process, so an address cached under an
// id stays valid exactly as long as that context lives.
unsigned long long current_context_id() {
  using CtxGetCurrentFn = CUresult (*)(CUcontext*);
  using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_static_pool on the current device.  It is looked up with
// cudaGetSymbolAddress the first time the device's current context calls, and again
// whenever that context has changed (after cudaDeviceReset the runtime creates a new
// primary context and loads the module again, at a new address).  Without a context id
// the address is looked up on every call.
rt_status static_pool_address(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RT_ERR_CUDA;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_static_pool_mutex);
  StaticPoolEntry& e = g_static_pool_addr[dev];
  if (ctx == 0 || e.ctx_id != ctx || e.addr == nullptr) {
    // The lookup makes the device's primary context current if no context was (a thread's
    // first runtime call), so the id is taken again after it.
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_pool) != cudaSuccess || p == nullptr) return RT_ERR_CUDA;
    e.addr = static_cast<float*>(p);
    e.ctx_id = current_context_id();
  }
  *out = e.addr;
  return RT_OK;
}

// Workspace of rt_attn_full_capture: the f16 copy of V, then the per-head max |v|.
size_t capture_workspace_bytes(const Dims& d) {
  return static_cast<size_t>(d.bh) * d.N * d.D * 2 + static_cast<size_t>(d.bh) * 4;
}

// Workspace of rt_build_block_mask_exact, in 256-byte aligned parts: the capture pass's
// workspace, an all-empty CSR row_ptr, the pass's m, Z_full, Z_kept and the per-tile
// log-sum-exp of every row.
struct ExactMaskLayout {
  size_t capture, row_ptr, m, zfull, zkept, block_lse, total;
};

ExactMaskLayout exact_mask_layout(const Dims& d) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t rows = static_cast<size_t>(d.bh) * d.N;
  ExactMaskLayout l;
  l.capture = 0;
  l.row_ptr = up(capture_workspace_bytes(d));
  l.m = l.row_ptr + up((static_cast<size_t>(d.bh) * d.n_blocks + 1) * 4);
  l.zfull = l.m + up(rows * 4);
  l.zkept = l.zfull + up(rows * 4);
  l.block_lse = l.zkept + up(rows * 4);
  l.total = l.block_lse + up(rows * rt::key_tiles(static_cast<int>(d.N)) * 4);
  return l;
}

// Workspace of rt_pair_query_blocks: the candidates of step 1 (none at block size 128).
size_t pairing_workspace_bytes(const Dims& d) {
  return d.bs == 64 ? static_cast<size_t>(d.bh) * d.n_blocks * rt::kPairCands * 2 : 0;
}

// One capture-kernel pass with its V prologue: the max |v| per head and the scaled f16 copy of
// V into `ws` (capture_workspace_bytes), then the capture kernel with the outputs set in `a`.
rt_status capture_pass(const Dims& d, const void* q, const void* k, const void* v, float scale,
                       const int32_t* row_ptr, const int32_t* col_idx, AttnArgs a, bool u16, void* ws,
                       cudaStream_t s) {
  const size_t per_head8 = static_cast<size_t>(d.N) * d.D / 8;  // D is a multiple of 16
  const size_t v16_bytes = static_cast<size_t>(d.bh) * per_head8 * 16;
  void* v16 = ws;
  uint32_t* amax = reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(ws) + v16_bytes);
  Maps m;
  // The output map is encoded on q when there is no output (the block-mass pass); it is unused.
  if (!make_maps(&m, d, q, k, v16, a.out != nullptr ? static_cast<const void*>(a.out) : q, rt::kBM, true))
    return RT_ERR_CUDA;
  const size_t per_head_blocks = (per_head8 + 255) / 256;
  const size_t want = (8 * static_cast<size_t>(sm_count()) + d.bh - 1) / d.bh;
  const dim3 cgrid(static_cast<unsigned>(std::max<size_t>(1, std::min(per_head_blocks, want))),
                   static_cast<unsigned>(d.bh));
  if (cudaMemsetAsync(amax, 0, static_cast<size_t>(d.bh) * 4, s) != cudaSuccess) return RT_ERR_CUDA;
  rt::v_absmax_kernel<<<cgrid, 256, 0, s>>>(static_cast<const uint4*>(v), per_head8, amax);
  if (launch_status() != RT_OK) return RT_ERR_CUDA;
  rt::convert_v_f16_kernel<<<cgrid, 256, 0, s>>>(static_cast<const uint4*>(v), static_cast<uint4*>(v16), per_head8,
                                                 amax);
  if (launch_status() != RT_OK) return RT_ERR_CUDA;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.v_amax = amax;
  a.N = static_cast<int>(d.N);
  a.d = static_cast<int>(d.d);
  a.n_blocks = static_cast<int>(d.n_blocks);
  a.n_heads = static_cast<int>(d.bh);
  a.scale_log2 = scale * rt::kLog2e;
  return dispatch_attention<true>(d, m, a, u16, s);
}

// The capture call behind rt_attn_full_capture (fp32 U) and rt_attn_full_capture_u16
// (f16 U with a per-row scale): exactly one of stat_u and stat_u16 is non-null.
rt_status full_capture_impl(const rt_shape* shape, const void* q, const void* k, const void* v, float scale,
                            const int32_t* row_ptr, const int32_t* col_idx, void* out, float* stat_m,
                            float* stat_zfull, float* stat_zkept, float* stat_u, uint16_t* stat_u16,
                            float* stat_u_scale, bool u16, void* workspace, size_t workspace_bytes,
                            cudaStream_t s) {
  Dims d;
  rt_status st = check_shape(shape, &d);
  if (st != RT_OK) return st;
  if (!q || !k || !v || !row_ptr || !col_idx || !out || !stat_m || !stat_zfull || !stat_zkept)
    return RT_ERR_INVALID_ARGUMENT;
  if (u16 ? (!stat_u16 || !stat_u_scale) : !stat_u) return RT_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(stat_u, 16) ||
      !aligned(stat_u16, 16) || !aligned(stat_u_scale, 4) || !aligned(row_ptr, 4) || !aligned(col_idx, 4) ||
      !aligned(stat_m, 4) || !aligned(stat_zfull, 4) || !aligned(stat_zkept, 4))
    return RT_ERR_INVALID_ARGUMENT;
  if (!scale_ok(scale)) return RT_ERR_INVALID_ARGUMENT;
  if (workspace && (!aligned(workspace, 16) || workspace_bytes < capture_workspace_bytes(d)))
    return RT_ERR_INVALID_ARGUMENT;
  // The PV products run on f16 P and an f16 copy of V scaled per head by a power of two
  // (workspace: the copy, then the per-head max |v|; the caller's, or from the pool).
  const bool own = workspace == nullptr;
  void* ws = workspace;
  if (own && !workspace_alloc(&ws, capture_workspace_bytes(d), s)) return RT_ERR_CUDA;
  AttnArgs a{};
  a.out_m = stat_m;
  a.out_zfull = stat_zfull;
  a.out_zkept = stat_zkept;
  a.out_u = stat_u;
  a.out_u16 = stat_u16;
  a.out_u_scale = stat_u_scale;
  a.out = static_cast<__nv_bfloat16*>(out);
  st = capture_pass(d, q, k, v, scale, row_ptr, col_idx, a, u16, ws, s);
  if (own && cudaFreeAsync(ws, s) != cudaSuccess && st == RT_OK) st = RT_ERR_CUDA;
  return st;
}

// The sparse call behind rt_attn_sparse_reshape and rt_attn_sparse_reshape_u16: with
// statistics, exactly one of stat_u and stat_u16 is non-null.
rt_status sparse_reshape_impl(const rt_shape* shape, const void* q, const void* k, const void* v, float scale,
                              const int32_t* row_ptr, const int32_t* col_idx, const int32_t* tile_blocks,
                              const float* stat_m, const float* stat_zfull, const float* stat_zkept,
                              const float* stat_u, const uint16_t* stat_u16, const float* stat_u_scale, bool u16,
                              void* out, cudaStream_t s) {
  Dims d;
  rt_status st = check_shape(shape, &d);
  if (st != RT_OK) return st;
  if (!q || !k || !v || !row_ptr || !col_idx || !out) return RT_ERR_INVALID_ARGUMENT;
  if (u16) {
    if (!stat_m || !stat_zfull || !stat_zkept || !stat_u16 || !stat_u_scale) return RT_ERR_INVALID_ARGUMENT;
  } else {
    const int nstats = (stat_m != nullptr) + (stat_zfull != nullptr) + (stat_zkept != nullptr) + (stat_u != nullptr);
    if (nstats != 0 && nstats != 4) return RT_ERR_INVALID_ARGUMENT;
  }
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(stat_u, 16) ||
      !aligned(stat_u16, 16) || !aligned(stat_u_scale, 4) || !aligned(row_ptr, 4) || !aligned(col_idx, 4) ||
      !aligned(tile_blocks, 4) || !aligned(stat_m, 4) || !aligned(stat_zfull, 4) || !aligned(stat_zkept, 4))
    return RT_ERR_INVALID_ARGUMENT;
  if (!scale_ok(scale)) return RT_ERR_INVALID_ARGUMENT;
  Maps m;
  if (!make_maps(&m, d, q, k, v, out, static_cast<int>(d.bs))) return RT_ERR_CUDA;
  AttnArgs a{};
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.tile_blocks = tile_blocks;
  a.stat_m = stat_m;
  a.stat_zfull = stat_zfull;
  a.stat_zkept = stat_zkept;
  a.stat_u = stat_u;
  a.stat_u16 = stat_u16;
  a.stat_u_scale = stat_u_scale;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.N = static_cast<int>(d.N);
  a.d = static_cast<int>(d.d);
  a.n_blocks = static_cast<int>(d.n_blocks);
  a.n_heads = static_cast<int>(d.bh);
  a.scale_log2 = scale * rt::kLog2e;
  return dispatch_attention<false>(d, m, a, u16, s);
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* rt_status_string(rt_status status) {
  switch (status) {
    case RT_OK: return "RT_OK";
    case RT_ERR_INVALID_ARGUMENT: return "RT_ERR_INVALID_ARGUMENT: bad pointer, size, keep count or alignment";
    case RT_ERR_UNSUPPORTED: return "RT_ERR_UNSUPPORTED: head dim, block size or size outside the supported set";
    case RT_ERR_CUDA: return "RT_ERR_CUDA: a CUDA call or kernel launch failed";
    case RT_ERR_TIMEOUT: return "RT_ERR_TIMEOUT: a kernel wait ran out and the kernel stopped";
  }
  return "unknown rt_status";
}

int32_t rt_abi_version(void) { return RT_ABI_VERSION; }

rt_status rt_build_block_mask(const rt_shape* shape, const void* q, const void* k, float scale, int32_t keep_blocks,
                              int32_t forced_prefix_tokens, int32_t* row_ptr, int32_t* col_idx, float* block_scores,
                              rt_stream_t stream) {
  Dims d;
  rt_status st = check_shape(shape, &d);
  if (st != RT_OK) return st;
  if (!q || !k || !row_ptr || !col_idx) return RT_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(row_ptr, 4) || !aligned(col_idx, 4) ||
      !aligned(block_scores, 4))
    return RT_ERR_INVALID_ARGUMENT;
  if (!scale_ok(scale) || forced_prefix_tokens < 0) return RT_ERR_INVALID_ARGUMENT;
  if (keep_blocks < 1 || keep_blocks > d.n_blocks) return RT_ERR_INVALID_ARGUMENT;
  const int64_t forced = std::min<int64_t>(d.n_blocks, (int64_t(forced_prefix_tokens) + d.bs - 1) / d.bs);
  if (forced > keep_blocks) return RT_ERR_INVALID_ARGUMENT;
  if (d.bh * d.n_blocks * keep_blocks > (int64_t(1) << 31) - 1) return RT_ERR_UNSUPPORTED;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* pooled = nullptr;
  const size_t bytes = sizeof(float) * 2 * d.bh * d.n_blocks * d.D;
  if (!workspace_alloc(reinterpret_cast<void**>(&pooled), bytes, s)) return RT_ERR_CUDA;
  st = mask_for_dim(d, q, k, scale, keep_blocks, forced_prefix_tokens, row_ptr, col_idx, block_scores, pooled, s);
  if (cudaFreeAsync(pooled, s) != cudaSuccess && st == RT_OK) st = RT_ERR_CUDA;
  return st;
}

rt_status rt_workspace_bytes(const rt_shape* shape, size_t* capture_bytes, size_t* pairing_bytes) {
  Dims d;
  rt_status st = check_shape(shape, &d);
  if (st != RT_OK) return st;
  if (capture_bytes) *capture_bytes = capture_workspace_bytes(d);
  if (pairing_bytes) *pairing_bytes = pairing_workspace_bytes(d);
  return RT_OK;
}

rt_status rt_attn_full_capture(const rt_shape* shape, const void* q, const void* k, const void* v, float scale,
                               const int32_t* row_ptr, const int32_t* col_idx, void* out, float* stat_m,
                               float* stat_zfull, float* stat_zkept, float* stat_u, void* workspace,
                               size_t workspace_bytes, rt_stream_t stream) {
  return full_capture_impl(shape, q, k, v, scale, row_ptr, col_idx, out, stat_m, stat_zfull, stat_zkept, stat_u,
                           nullptr, nullptr, false, workspace, workspace_bytes,
                           reinterpret_cast<cudaStream_t>(stream));
}

rt_status rt_attn_full_capture_u16(const rt_shape* shape, const void* q, const void* k, const void* v, float scale,
                                   const int32_t* row_ptr, const int32_t* col_idx, void* out, float* stat_m,
                                   float* stat_zfull, float* stat_zkept, uint16_t* stat_u16, float* stat_u_scale,
                                   void* workspace, size_t workspace_bytes, rt_stream_t stream) {
  return full_capture_impl(shape, q, k, v, scale, row_ptr, col_idx, out, stat_m, stat_zfull, stat_zkept, nullptr,
                           stat_u16, stat_u_scale, true, workspace, workspace_bytes,
                           reinterpret_cast<cudaStream_t>(stream));
}

rt_status rt_attn_sparse_reshape(const rt_shape* shape, const void* q, const void* k, const void* v, float scale,
                                 const int32_t* row_ptr, const int32_t* col_idx, const int32_t* tile_blocks,
                                 const float* stat_m, const float* stat_zfull, const float* stat_zkept,
                                 const float* stat_u, void* out, rt_stream_t stream) {
  return sparse_reshape_impl(shape, q, k, v, scale, row_ptr, col_idx, tile_blocks, stat_m, stat_zfull, stat_zkept,
                             stat_u, nullptr, nullptr, false, out, reinterpret_cast<cudaStream_t>(stream));
}

rt_status rt_attn_sparse_reshape_u16(const rt_shape* shape, const void* q, const void* k, const void* v, float scale,
                                     const int32_t* row_ptr, const int32_t* col_idx, const int32_t* tile_blocks,
                                     const float* stat_m, const float* stat_zfull, const float* stat_zkept,
                                     const uint16_t* stat_u16, const float* stat_u_scale, void* out,
                                     rt_stream_t stream) {
  return sparse_reshape_impl(shape, q, k, v, scale, row_ptr, col_idx, tile_blocks, stat_m, stat_zfull, stat_zkept,
                             nullptr, stat_u16, stat_u_scale, true, out, reinterpret_cast<cudaStream_t>(stream));
}

rt_status rt_pair_query_blocks(const rt_shape* shape, const int32_t* row_ptr, const int32_t* col_idx,
                               int32_t* tile_blocks, void* workspace, size_t workspace_bytes, rt_stream_t stream) {
  Dims d;
  rt_status st = check_shape(shape, &d);
  if (st != RT_OK) return st;
  if (!row_ptr || !col_idx || !tile_blocks) return RT_ERR_INVALID_ARGUMENT;
  if (!aligned(row_ptr, 4) || !aligned(col_idx, 4) || !aligned(tile_blocks, 4)) return RT_ERR_INVALID_ARGUMENT;
  if (workspace && (!aligned(workspace, 16) || workspace_bytes < pairing_workspace_bytes(d)))
    return RT_ERR_INVALID_ARGUMENT;
  const int nb = static_cast<int>(d.n_blocks);
  const int n_tiles = rt::query_tiles(static_cast<int>(d.N));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d.bs != 64) {  // one query block per tile: the identity table
    rt::pair_match_kernel<<<static_cast<unsigned>(d.bh), rt::kPairThreads, 0, s>>>(nullptr, nb, n_tiles,
                                                                                 static_cast<int>(d.bs), tile_blocks);
    return launch_status();
  }
  // Candidates of every query block go through a workspace (int16 [B*H][n_blocks][8]): the
  // caller's, or from the pool.
  const size_t cand_smem = rt::pair_candidates_smem_bytes(nb), match_smem = rt::pair_match_smem_bytes(nb);
  // Block i's kept-set bitmap lives in registers, in the smallest of these word counts that holds it.
  const int words = (nb + 31) / 32;
  auto cand_kernel = words <= 8    ? rt::pair_candidates_kernel<8>
                     : words <= 12 ? rt::pair_candidates_kernel<12>
                     : words <= 16 ? rt::pair_candidates_kernel<16>
                     : words <= 32 ? rt::pair_candidates_kernel<32>
                                   : rt::pair_candidates_kernel<64>;
  static_assert(kMaxBlocks <= 64 * 32, "pairing bitmap words");
  if (cudaFuncSetAttribute(cand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(cand_smem)) != cudaSuccess ||
      cudaFuncSetAttribute(rt::pair_match_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(match_smem)) != cudaSuccess)
    return RT_ERR_CUDA;
  const bool own = workspace == nullptr;
  int16_t* cand = static_cast<int16_t*>(workspace);
  if (own && !workspace_alloc(reinterpret_cast<void**>(&cand), pairing_workspace_bytes(d), s)) return RT_ERR_CUDA;
  dim3 grid(static_cast<unsigned>((nb + rt::kCandBlocks - 1) / rt::kCandBlocks), static_cast<unsigned>(d.bh));
  cand_kernel<<<grid, rt::kPairThreads, cand_smem, s>>>(row_ptr, col_idx, nb, cand);
  st = launch_status();
  if (st == RT_OK) {
    rt::pair_match_kernel<<<static_cast<unsigned>(d.bh), rt::kPairThreads, match_smem, s>>>(cand, nb, n_tiles, 64,
                                                                                          tile_blocks);
    st = launch_status();
  }
  if (own && cudaFreeAsync(cand, s) != cudaSuccess && st == RT_OK) st = RT_ERR_CUDA;
  return st;
}

rt_status rt_build_block_mask_static(const rt_shape* shape, const void* q, const void* k, float scale,
                                     int32_t keep_blocks, int32_t forced_prefix_tokens, int32_t* row_ptr,
                                     int32_t* col_idx, float* block_scores, rt_stream_t stream) {
  Dims d;
  rt_status st = check_shape(shape, &d);
  if (st != RT_OK) return st;
  if (!q || !k || !row_ptr || !col_idx) return RT_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(row_ptr, 4) || !aligned(col_idx, 4) ||
      !aligned(block_scores, 4))
    return RT_ERR_INVALID_ARGUMENT;
  if (!scale_ok(scale) || forced_prefix_tokens < 0) return RT_ERR_INVALID_ARGUMENT;
  if (keep_blocks < 1 || keep_blocks > d.n_blocks) return RT_ERR_INVALID_ARGUMENT;
  const int64_t forced = std::min<int64_t>(d.n_blocks, (int64_t(forced_prefix_tokens) + d.bs - 1) / d.bs);
  if (forced > keep_blocks) return RT_ERR_INVALID_ARGUMENT;
  if (d.bh * d.n_blocks * keep_blocks > (int64_t(1) << 31) - 1) return RT_ERR_UNSUPPORTED;
  if (static_cast<size_t>(2 * d.bh * d.n_blocks * d.D) > kStaticPoolFloats) return RT_ERR_UNSUPPORTED;
  float* pooled = nullptr;
  st = static_pool_address(&pooled);
  if (st != RT_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return mask_for_dim(d, q, k, scale, keep_blocks, forced_prefix_tokens, row_ptr, col_idx, block_scores, pooled, s);
}

rt_status rt_exact_mask_workspace_bytes(const rt_shape* shape, size_t* bytes) {
  Dims d;
  rt_status st = check_shape(shape, &d);
  if (st != RT_OK) return st;
  if (!bytes) return RT_ERR_INVALID_ARGUMENT;
  *bytes = exact_mask_layout(d).total;
  return RT_OK;
}

rt_status rt_build_block_mask_exact(const rt_shape* shape, const void* q, const void* k, const void* v, float scale,
                                    int32_t keep_blocks, int32_t forced_prefix_tokens, int32_t* row_ptr,
                                    int32_t* col_idx, float* block_mass, void* workspace, size_t workspace_bytes,
                                    rt_stream_t stream) {
  Dims d;
  rt_status st = check_shape(shape, &d);
  if (st != RT_OK) return st;
  if (!q || !k || !v || !row_ptr || !col_idx) return RT_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(row_ptr, 4) || !aligned(col_idx, 4) ||
      !aligned(block_mass, 4))
    return RT_ERR_INVALID_ARGUMENT;
  if (!scale_ok(scale) || forced_prefix_tokens < 0) return RT_ERR_INVALID_ARGUMENT;
  if (keep_blocks < 1 || keep_blocks > d.n_blocks) return RT_ERR_INVALID_ARGUMENT;
  const int64_t forced = std::min<int64_t>(d.n_blocks, (int64_t(forced_prefix_tokens) + d.bs - 1) / d.bs);
  if (forced > keep_blocks) return RT_ERR_INVALID_ARGUMENT;
  if (d.bh * d.n_blocks * keep_blocks > (int64_t(1) << 31) - 1) return RT_ERR_UNSUPPORTED;
  const ExactMaskLayout l = exact_mask_layout(d);
  if (workspace && (!aligned(workspace, 256) || workspace_bytes < l.total)) return RT_ERR_INVALID_ARGUMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool own = workspace == nullptr;
  void* ws = workspace;
  if (own && !workspace_alloc(&ws, l.total, s)) return RT_ERR_CUDA;
  unsigned char* base = static_cast<unsigned char*>(ws);
  int32_t* empty_rp = reinterpret_cast<int32_t*>(base + l.row_ptr);
  float* m = reinterpret_cast<float*>(base + l.m);
  float* zf = reinterpret_cast<float*>(base + l.zfull);
  float* zk = reinterpret_cast<float*>(base + l.zkept);
  float* lse = reinterpret_cast<float*>(base + l.block_lse);
  // Pass 1: full attention statistics of every row with no key block kept (every tile goes
  // to the masked sum; O and U are not stored), and each row's per-tile log-sum-exp.
  st = cudaMemsetAsync(empty_rp, 0, (static_cast<size_t>(d.bh) * d.n_blocks + 1) * 4, s) == cudaSuccess
           ? RT_OK
           : RT_ERR_CUDA;
  if (st == RT_OK) {
    AttnArgs a{};
    a.out_m = m;
    a.out_zfull = zf;
    a.out_zkept = zk;
    a.out_block_lse = lse;
    st = capture_pass(d, q, k, v, scale, empty_rp, empty_rp, a, false, base + l.capture, s);
  }
  // Pass 2: block masses from the log-sum-exps, then the top-k selection per query block.
  if (st == RT_OK) {
    const size_t smem = rt::mass_select_smem_bytes(static_cast<int>(d.n_blocks));
    if (cudaFuncSetAttribute(rt::mass_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess) {
      st = RT_ERR_CUDA;
    } else {
      dim3 grid(static_cast<unsigned>((d.n_blocks + rt::kSelWarps - 1) / rt::kSelWarps),
                static_cast<unsigned>(d.bh));
      rt::mass_select_kernel<<<grid, 32 * rt::kSelWarps, smem, s>>>(
          lse, m, zf, static_cast<int>(d.N), static_cast<int>(d.n_blocks), static_cast<int>(d.bs), keep_blocks,
          forced_prefix_tokens, row_ptr, col_idx, block_mass);
      st = launch_status();
    }
  }
  if (own && cudaFreeAsync(ws, s) != cudaSuccess && st == RT_OK) st = RT_ERR_CUDA;
  return st;
}

rt_status rt_hilbert_order(int32_t prefix_tokens, int32_t frames, int32_t grid_h, int32_t grid_w, int32_t* perm) {
  if (!perm || prefix_tokens < 0 || frames < 1 || grid_h < 1 || grid_w < 1) return RT_ERR_INVALID_ARGUMENT;
  if (grid_h > (1 << 15) || grid_w > (1 << 15)) return RT_ERR_UNSUPPORTED;
  const int64_t cells = int64_t(grid_h) * grid_w;
  if (prefix_tokens + frames * cells > (int64_t(1) << 31) - 1) return RT_ERR_UNSUPPORTED;
  int k = 0;
  while ((1 << k) < std::max(grid_h, grid_w)) ++k;
  // The grid's cells in the order of the enclosing square's curve (cells outside are skipped).
  std::vector<std::pair<uint64_t, int32_t>> order(static_cast<size_t>(cells));
  for (int32_t y = 0; y < grid_h; ++y)
    for (int32_t x = 0; x < grid_w; ++x)
      order[static_cast<size_t>(y) * grid_w + x] = {rt::hilbert_index(k, x, y), y * grid_w + x};
  std::sort(order.begin(), order.end());
  for (int32_t t = 0; t < prefix_tokens; ++t) perm[t] = t;
  for (int32_t f = 0; f < frames; ++f) {
    const int64_t base = prefix_tokens + f * cells;
    for (int64_t c = 0; c < cells; ++c) perm[base + c] = static_cast<int32_t>(base + order[static_cast<size_t>(c)].second);
  }
  return RT_OK;
}

rt_status rt_permute_tokens(const rt_shape* shape, const void* src, const int32_t* perm, int32_t inverse, void* dst,
                            rt_stream_t stream) {
  Dims d;
  rt_status st = check_shape(shape, &d);
  if (st != RT_OK) return st;
  if (!src || !perm || !dst || src == dst) return RT_ERR_INVALID_ARGUMENT;
  if (!aligned(src, 16) || !aligned(dst, 16) || !aligned(perm, 4)) return RT_ERR_INVALID_ARGUMENT;
  const int chunks = static_cast<int>(d.D / 8);  // 16-byte chunks of a bf16 row
  const size_t per_head = static_cast<size_t>(d.N) * chunks;
  const dim3 grid(static_cast<unsigned>((per_head + 255) / 256), static_cast<unsigned>(d.bh));
  rt::permute_rows_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), perm, static_cast<uint4*>(dst), static_cast<int>(d.N), chunks,
      inverse ? 1 : 0);
  return launch_status();
}

rt_status rt_take_device_error(int32_t* code) {
  if (code == nullptr) return RT_ERR_INVALID_ARGUMENT;
  if (cudaDeviceSynchronize() != cudaSuccess) return RT_ERR_CUDA;
  int32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, rt::g_device_status, sizeof(v)) != cudaSuccess) return RT_ERR_CUDA;
  if (cudaMemcpyToSymbol(rt::g_device_status, &zero, sizeof(zero)) != cudaSuccess) return RT_ERR_CUDA;
  *code = v;
  return RT_OK;
}

rt_status rt_selftest_exp2_poly(const float* x, float* y, int32_t n, rt_stream_t stream) {
  if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return RT_ERR_INVALID_ARGUMENT;
  if (!aligned(x, 4) || !aligned(y, 4)) return RT_ERR_INVALID_ARGUMENT;
  if (n == 0) return RT_OK;
  const int pairs = (n + 1) / 2;
  rt::exp2_poly_selftest_kernel<<<(pairs + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return launch_status();
}

rt_status rt_selftest_wait_timeout(int64_t timeout_ns, rt_stream_t stream) {
  if (timeout_ns <= 0 || timeout_ns > 10000000000ll) return RT_ERR_INVALID_ARGUMENT;
  rt::wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(timeout_ns));
  return launch_status();
}

}  // extern "C"
