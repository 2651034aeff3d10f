// dsa_api.cu -- the C ABI of include/dsa.h: host-side argument checks, launch
// geometry and the dsa_forward orchestration over the three kernels.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <cmath>
#include <mutex>
#include <vector>

#include "../../include/dsa.h"
#include "ptx.cuh"
#include "topk.cuh"
#include "indexer.cuh"
#include "sparse_mla.cuh"
#include "indexer_kl.cuh"
#include "mha_prefill.cuh"

using namespace dsa;

namespace {

constexpr int kDIdx = 128, kMaxK = 2048;

std::atomic<uint64_t> g_timeout_ns{2000000000ull};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dsa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Validated geometry shared by every entry point.
struct Geometry {
  int layout, batch, max_ctx, page_size, num_pages, max_pages, q_per_seq, num_q;
  int row_begin, row_count;  // window of rows per sequence
  const int32_t* block_table;
  const int32_t* seqlens;
  const int32_t* q_start;    // ragged query rows ([batch + 1], device) or nullptr
  int64_t cache_rows;  // rows of each per-token cache array
};

dsa_status_t check_geometry(const dsa_kv_desc_t* kv, const dsa_q_desc_t* q, Geometry* g) {
  if (!kv || !q) return DSA_ERR_INVALID_ARG;
  if (kv->batch < 1 || kv->max_ctx < 1 || q->q_per_seq < 1) return DSA_ERR_INVALID_ARG;
  if (q->q_start) {  // ragged: every sequence has at most q_per_seq rows
    if (q->num_q < 0 || (int64_t)q->num_q > (int64_t)kv->batch * q->q_per_seq)
      return DSA_ERR_INVALID_ARG;
  } else if ((int64_t)kv->batch * q->q_per_seq != q->num_q) {
    return DSA_ERR_INVALID_ARG;
  }
  if (q->q_per_seq > kv->max_ctx) return DSA_ERR_INVALID_ARG;
  if (q->row_begin < 0 || q->row_begin >= q->q_per_seq || q->row_count < 0 ||
      q->row_count > q->q_per_seq - q->row_begin)
    return DSA_ERR_INVALID_ARG;
  g->row_begin = q->row_begin;
  g->row_count = q->row_count ? q->row_count : q->q_per_seq - q->row_begin;
  g->layout = kv->layout;
  g->batch = kv->batch;
  g->max_ctx = kv->max_ctx;
  g->q_per_seq = q->q_per_seq;
  g->num_q = q->num_q;
  g->q_start = q->q_start;
  g->seqlens = kv->seqlens;
  g->block_table = nullptr;
  g->page_size = 0;
  g->num_pages = 0;
  g->max_pages = 0;
  if (kv->layout == DSA_KV_CONTIGUOUS) {
    g->cache_rows = (int64_t)kv->batch * kv->max_ctx;
  } else if (kv->layout == DSA_KV_PAGED) {
    if (!kv->block_table || kv->num_pages < 1 || kv->max_pages < 1) return DSA_ERR_INVALID_ARG;
    if (kv->page_size < 64 || kv->page_size % 64 != 0) return DSA_ERR_UNSUPPORTED_SHAPE;
    if ((int64_t)kv->max_pages * kv->page_size < kv->max_ctx) return DSA_ERR_INVALID_ARG;
    g->block_table = kv->block_table;
    g->page_size = kv->page_size;
    g->num_pages = kv->num_pages;
    g->max_pages = kv->max_pages;
    g->cache_rows = (int64_t)kv->num_pages * kv->page_size;
  } else {
    return DSA_ERR_INVALID_ARG;
  }
  if (g->cache_rows >= (1ll << 31)) return DSA_ERR_UNSUPPORTED_SHAPE;
  return DSA_OK;
}

// Per-device state: kernel attributes belong to each device's context, so a
// process that drives several GPUs sets them (and reads the SM count) on each.
constexpr int kMaxDevices = 64;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

int num_sms() {
  static std::atomic<int> sms[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return 148;
  int n = sms[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 2)
      n = 148;
    sms[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Runs `fn` (which returns a cudaError_t) once per device and remembers its result.
struct DeviceOnce {
  std::mutex mu;
  bool done[kMaxDevices] = {};
  cudaError_t err[kMaxDevices] = {};
};

template <typename Fn>
cudaError_t once_per_device(DeviceOnce& o, Fn&& fn) {
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(o.mu);
  if (!o.done[dev]) {
    o.err[dev] = fn();
    o.done[dev] = true;
  }
  return o.err[dev];
}

// ---- top-k launch ------------------------------------------------------------------
dsa_status_t launch_topk(const float* scores, int64_t ld, const Geometry& g, int row_begin,
                         int row_count, int k, int32_t* idx, cudaStream_t stream,
                         int tile_stride = 1, float* kth_out = nullptr) {
  static DeviceOnce once;
  const cudaError_t attr_err = once_per_device(once, [] {
    return cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kTopkSmemBytes);
  });
  if (attr_err != cudaSuccess) return DSA_ERR_CUDA;
  TopkParams p{scores, ld, g.seqlens, g.max_ctx, g.q_per_seq, row_begin, row_count, g.batch, k,
               idx, tile_stride, kth_out, g.q_start, g.num_q};
  const int64_t grid = (int64_t)g.batch * row_count;
  if (grid == 0) return DSA_OK;
  topk_kernel<<<(unsigned)grid, kTopkThreads, kTopkSmemBytes, stream>>>(p);
  return cuda_status(cudaGetLastError());
}

// ---- split top-k (long rows swept by several CTAs) ----------------------------------
// Scratch of the split path for `rows` window rows: each row's candidate keys and
// positions (kCandCap each), then the rows' candidate counts and threshold keys.
size_t split_topk_bytes(int64_t rows) {
  return align256((size_t)rows * kCandCap * 8) + 2 * align256((size_t)rows * 4);
}

// dsa_forward's choice between the two selections. Measured on B200 (paged 128K
// decode, 256 rows, CUDA events around the selection inside the step): the split
// path takes 85 us (three kernels) against 63 us for one CTA per row. Each of the
// three is bound by fixed latency
// (short-lived sweep CTAs in waves, and the block-wide radix passes of the threshold
// and of the selection), so the forward keeps one CTA per row; the split path stays
// available through dsa_topk_ws.
constexpr bool kForwardSplitTopk = false;

// Whether the split path applies: some row may hold more than 4k keys (else the
// one-CTA kernel has nothing to split) and every row fits the selection bitmaps.
bool split_topk_applies(const Geometry& g, int k) {
  return g.max_ctx > 4 * k && g.max_ctx <= kCandMaxWords * 32;
}

dsa_status_t launch_topk_split(const float* scores, int64_t ld, const Geometry& g,
                               int row_begin, int row_count, int k, int32_t* idx,
                               cudaStream_t stream, void* scratch) {
  static DeviceOnce once;
  const cudaError_t attr_err = once_per_device(once, [] {
    return cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSelectSmemBytes);
  });
  if (attr_err != cudaSuccess) return DSA_ERR_CUDA;
  const int64_t rows = (int64_t)g.batch * row_count;
  if (rows == 0) return DSA_OK;
  uint8_t* ws = reinterpret_cast<uint8_t*>(scratch);
  SplitParams p{};
  p.scores = scores;
  p.ld = ld;
  p.seqlens = g.seqlens;
  p.q_start = g.q_start;
  p.num_q = g.num_q;
  p.max_ctx = g.max_ctx;
  p.q_per_seq = g.q_per_seq;
  p.row_begin = row_begin;
  p.row_count = row_count;
  p.batch = g.batch;
  p.k = k;
  p.nchunk = (g.max_ctx + kSplitChunk - 1) / kSplitChunk;
  p.cand_key = reinterpret_cast<uint32_t*>(ws);
  p.cand_pos = reinterpret_cast<int32_t*>(ws + (size_t)rows * kCandCap * 4);
  p.cand_cnt = reinterpret_cast<uint32_t*>(ws + align256((size_t)rows * kCandCap * 8));
  p.thr_key = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(p.cand_cnt) +
                                          align256((size_t)rows * 4));
  p.idx = idx;
  topk_threshold_kernel<<<(unsigned)rows, kThresholdThreads, 0, stream>>>(p);
  dsa_status_t st = cuda_status(cudaGetLastError());
  if (st != DSA_OK) return st;
  topk_sweep_kernel<<<(unsigned)(rows * p.nchunk), kTopkThreads, 0, stream>>>(p);
  st = cuda_status(cudaGetLastError());
  if (st != DSA_OK) return st;
  topk_select_kernel<<<(unsigned)rows, kTopkThreads, kSelectSmemBytes, stream>>>(p);
  return cuda_status(cudaGetLastError());
}

// ---- TMA tensor maps ---------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

// 2-D row-major tensor [rows][cols] with 128-byte swizzled boxes of box_rows x box_cols.
dsa_status_t make_tmap_2d(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                          int elem_bytes, uint64_t cols, uint64_t rows, uint32_t box_cols,
                          uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return DSA_ERR_CUDA;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(tm, dtype, 2, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DSA_OK : DSA_ERR_CUDA;
}

// ---- indexer launch -----------------------------------------------------------------
// Candidate output of the indexer's filter mode (see IndexerParams).
struct IdxFilter {
  const float* thr = nullptr;
  uint32_t* cand_key = nullptr;
  int32_t* cand_pos = nullptr;
  uint32_t* cand_cnt = nullptr;
  int cand_cap = 0;
};

dsa_status_t launch_indexer(const void* q_idx, const float* w, const void* k_idx,
                            const float* k_scale, const Geometry& g, float* scores, int64_t ld,
                            int row_begin, int row_count, cudaStream_t stream,
                            int tile_stride = 1, const IdxFilter& filt = IdxFilter()) {
  static DeviceOnce once;
  const cudaError_t attr_err = once_per_device(once, [] {
    cudaError_t e = cudaFuncSetAttribute(indexer_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kIdxSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(indexer_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kIdxSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(indexer_kernel<false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kIdxLeanSmemBytes);
    return e;
  });
  if (attr_err != cudaSuccess) return DSA_ERR_CUDA;
  CUtensorMap tm;
  dsa_status_t st = make_tmap_2d(&tm, k_idx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kDIdx,
                                 (uint64_t)g.cache_rows, kDIdx, 64);
  if (st != DSA_OK) return st;
  IndexerParams p{};
  p.q_idx = reinterpret_cast<const __nv_bfloat16*>(q_idx);
  p.k_idx = reinterpret_cast<const uint8_t*>(k_idx);
  p.cache_rows = g.cache_rows;
  p.w = w;
  p.k_scale = k_scale;
  p.block_table = g.block_table;
  p.seqlens = g.seqlens;
  p.scores = scores;
  p.ld = ld;
  p.batch = g.batch;
  p.max_ctx = g.max_ctx;
  p.q_per_seq = g.q_per_seq;
  p.paged = g.layout == DSA_KV_PAGED;
  p.page_size = g.page_size;
  p.max_pages = g.max_pages;
  p.num_pages = g.num_pages;
  p.row_begin = row_begin;
  p.row_count = row_count;
  p.G = std::min(4, row_count);
  p.groups_per_seq = (row_count + p.G - 1) / p.G;
  p.num_groups = g.batch * p.groups_per_seq;
  p.tile_stride = tile_stride;
  p.thr = filt.thr;
  p.cand_key = filt.cand_key;
  p.cand_pos = filt.cand_pos;
  p.cand_cnt = filt.cand_cnt;
  p.cand_cap = filt.cand_cap;
  p.q_start = g.q_start;
  p.num_q = g.num_q;
  p.timeout_ns = g_timeout_ns.load();
  // every CTA takes an equal share of all key tiles (at most one CTA per tile)
  const int64_t max_tiles = (int64_t)p.num_groups * ((g.max_ctx + kIdxTile - 1) / kIdxTile);
  const int grid = (int)std::min<int64_t>(max_tiles, num_sms());
  if (p.thr) {
    indexer_kernel<true><<<grid, kIdxThreads, kIdxSmemBytes, stream>>>(p, tm);
  } else if (p.G <= 2) {
    // decode groups: two lean CTAs per SM (each takes an equal share as well)
    const int grid2 = (int)std::min<int64_t>(max_tiles, 2 * (int64_t)num_sms());
    indexer_kernel<false, true><<<grid2, kIdxLeanThreads, kIdxLeanSmemBytes, stream>>>(p, tm);
  } else {
    indexer_kernel<false><<<grid, kIdxThreads, kIdxSmemBytes, stream>>>(p, tm);
  }
  return cuda_status(cudaGetLastError());
}

// ---- sparse MLA launch --------------------------------------------------------------
// How the rows of one call are spread over clusters. A call's clusters run in waves
// of (SMs / 2) clusters; when the last wave is at most half full, its rows are split
// into as many key segments as fill it (at least 6 key blocks each, at most
// kMlaMaxSeg, and only as many as the scratch holds), and merged afterwards.
struct MlaSplit {
  int64_t n_whole = 0, n_split = 0;
  int nseg = 1, seg_keys = 0;
};
constexpr size_t kMlaPartBytes = (size_t)kMlaHeads * kMlaDv * 4 + kMlaHeads * 4;

MlaSplit plan_mla_split(int64_t rows, int k, size_t scratch_bytes) {
  MlaSplit sp;
  sp.n_whole = rows;
  sp.seg_keys = k;
  const int64_t wave = num_sms() / 2;
  if (wave < 2 || rows <= 0) return sp;
  const int64_t tail = rows % wave;
  const int nb = (k + kMlaBlk - 1) / kMlaBlk;
  if (tail == 0) return sp;
  int s = (int)std::min<int64_t>(wave / tail, kMlaMaxSeg);
  s = std::min(s, nb / 6);
  while (s >= 2 && (size_t)tail * s * kMlaPartBytes > scratch_bytes) --s;
  if (s < 2) return sp;
  const int bps = (nb + s - 1) / s;  // blocks per segment; every segment non-empty
  sp.nseg = (nb + bps - 1) / bps;
  if (sp.nseg < 2) return sp;
  sp.seg_keys = bps * kMlaBlk;
  sp.n_whole = rows - tail;
  sp.n_split = tail;
  return sp;
}

// `scratch` (256-B aligned, may be null) holds the segments' partial outputs.
dsa_status_t launch_sparse_mla(const void* q, const void* kv_cache, const Geometry& g,
                               const int32_t* idx, int k, float scale, void* out, float* lse,
                               cudaStream_t stream, void* scratch = nullptr,
                               size_t scratch_bytes = 0) {
  static DeviceOnce once;
  const cudaError_t attr_err = once_per_device(once, [] {
    return cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kMlaSmemBytes);
  });
  if (attr_err != cudaSuccess) return DSA_ERR_CUDA;
  // the latent cache as [cache_rows][576] bf16, gathered 64 dims of one row per box row
  CUtensorMap tm;
  dsa_status_t st = make_tmap_2d(&tm, kv_cache, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kMlaDqk,
                                 (uint64_t)g.cache_rows, 64, 1);
  if (st != DSA_OK) return st;
  MlaParams p{};
  p.kv = reinterpret_cast<const uint8_t*>(kv_cache);
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.idx = idx;
  p.block_table = g.block_table;
  p.seqlens = g.seqlens;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.k = k;
  p.batch = g.batch;
  p.max_ctx = g.max_ctx;
  p.q_per_seq = g.q_per_seq;
  p.paged = g.layout == DSA_KV_PAGED;
  p.page_size = g.page_size;
  p.max_pages = g.max_pages;
  p.num_pages = g.num_pages;
  p.cache_rows = g.cache_rows;
  p.row_begin = g.row_begin;
  p.row_count = g.row_count;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load();
  p.q_start = g.q_start;
  p.num_q = g.num_q;
  const int64_t rows = (int64_t)g.batch * g.row_count;
  if (rows == 0) return DSA_OK;
  const MlaSplit sp = plan_mla_split(rows, k, scratch ? scratch_bytes : 0);
  p.n_whole = sp.n_whole;
  p.nseg = sp.nseg;
  p.seg_keys = sp.seg_keys;
  const int64_t slots = sp.n_split * sp.nseg;
  if (slots > 0) {
    p.part_o = reinterpret_cast<float*>(scratch);
    p.part_lse = p.part_o + slots * kMlaHeads * kMlaDv;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(2 * (sp.n_whole + slots)), 1, 1);
  cfg.blockDim = dim3(kMlaThreads, 1, 1);
  cfg.dynamicSmemBytes = kMlaSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  st = cuda_status(cudaLaunchKernelEx(&cfg, sparse_mla_kernel, p, tm));
  if (st != DSA_OK || slots == 0) return st;
  MlaCombineParams c{};
  c.part_o = p.part_o;
  c.part_lse = p.part_lse;
  c.out = p.out;
  c.lse = lse;
  c.n_whole = sp.n_whole;
  c.nseg = sp.nseg;
  c.row_begin = g.row_begin;
  c.row_count = g.row_count;
  c.q_per_seq = g.q_per_seq;
  c.q_start = g.q_start;
  c.seqlens = g.seqlens;
  c.num_q = g.num_q;
  c.max_ctx = g.max_ctx;
  mla_combine_kernel<<<dim3((unsigned)sp.n_split, kMlaHeads / 8), 256, 0, stream>>>(c);
  return cuda_status(cudaGetLastError());
}

// ---- indexer KL launch -------------------------------------------------------------
dsa_status_t launch_indexer_kl(const void* q, const void* kv_cache, const Geometry& g,
                               const int32_t* idx, int k, float scale, const float* lse,
                               const float* scores, int64_t ld, float* kl, cudaStream_t stream) {
  static DeviceOnce once;
  const cudaError_t attr_err = once_per_device(once, [] {
    return cudaFuncSetAttribute(indexer_kl_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kKlSmemBytes);
  });
  if (attr_err != cudaSuccess) return DSA_ERR_CUDA;
  KlParams p{};
  p.kv = reinterpret_cast<const uint8_t*>(kv_cache);
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.idx = idx;
  p.lse = lse;
  p.scores = scores;
  p.block_table = g.block_table;
  p.seqlens = g.seqlens;
  p.kl = kl;
  p.ld = ld;
  p.k = k;
  p.batch = g.batch;
  p.max_ctx = g.max_ctx;
  p.q_per_seq = g.q_per_seq;
  p.row_begin = g.row_begin;
  p.row_count = g.row_count;
  p.paged = g.layout == DSA_KV_PAGED;
  p.page_size = g.page_size;
  p.max_pages = g.max_pages;
  p.num_pages = g.num_pages;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load();
  p.q_start = g.q_start;
  p.num_q = g.num_q;
  const int64_t grid = (int64_t)g.batch * g.row_count;
  if (grid == 0) return DSA_OK;
  indexer_kl_kernel<<<(unsigned)grid, kKlThreads, kKlSmemBytes, stream>>>(p);
  return cuda_status(cudaGetLastError());
}

// ---- dsa_forward workspace plan --------------------------------------------------------
constexpr int64_t kScoreBudgetBytes = 2ll << 30;  // bound on one chunk of score rows

struct ForwardPlan {
  int64_t ld;           // score row stride
  int chunk_rows;       // query rows per sequence per chunk
  size_t idx_bytes;     // selected indices (0 when the caller provides idx_out)
  size_t score_bytes;   // one chunk of score rows
};


ForwardPlan plan_forward(const Geometry& g, int k, bool need_idx) {
  ForwardPlan f;
  f.ld = (int64_t)(g.max_ctx + kIdxTile - 1) / kIdxTile * kIdxTile;
  const int64_t row_bytes = f.ld * 4 * g.batch;  // one row index across all sequences
  int64_t rows = std::max<int64_t>(1, kScoreBudgetBytes / row_bytes);
  if (rows >= g.row_count) {
    rows = g.row_count;
  } else if (rows >= 4) {
    rows &= ~int64_t(3);  // whole groups of 4 rows per indexer MMA
  }
  f.chunk_rows = (int)rows;
  f.idx_bytes = need_idx ? align256((size_t)g.num_q * k * 4) : 0;
  f.score_bytes = align256((size_t)f.chunk_rows * row_bytes);
  return f;
}

// ---- MHA mode: up-projection, selection mask, masked MHA --------------------------------
// 3-D row-major tensor [d2][d1][d0] with 128-byte swizzled boxes.
dsa_status_t make_tmap_3d(CUtensorMap* tm, const void* base, CUtensorMapDataType dtype,
                          int elem_bytes, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                          uint32_t b1, uint32_t b2) {
  auto enc = tensor_map_encoder();
  if (!enc) return DSA_ERR_CUDA;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * elem_bytes, d0 * d1 * elem_bytes};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(tm, dtype, 3, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DSA_OK : DSA_ERR_CUDA;
}

struct MhaPlan {
  int key_tiles;
  int64_t ctx_pad;      // key slots per (sequence, head) in the decompressed tensors
  int64_t mask_ld;      // words per selection-mask row
  size_t kn_bytes, kr_bytes, v_bytes, mask_bytes;
};

MhaPlan plan_mha(const Geometry& g) {
  MhaPlan m;
  m.key_tiles = (g.max_ctx + kMhaTile - 1) / kMhaTile;
  m.ctx_pad = (int64_t)m.key_tiles * kMhaTile;
  m.mask_ld = (int64_t)m.key_tiles * 4;
  m.kn_bytes = align256((size_t)g.batch * kMhaHeads * m.ctx_pad * kMhaDn * 2);
  m.kr_bytes = align256((size_t)g.batch * m.ctx_pad * kMhaDr * 2);
  m.v_bytes = align256((size_t)g.batch * kMhaHeads * m.ctx_pad * kMhaDv * 2);
  m.mask_bytes = align256((size_t)g.num_q * m.mask_ld * 4);
  return m;
}

// every decompressed row index of the tensor maps must fit in int32
bool mha_fits(const Geometry& g, int64_t ctx_pad) {
  return (int64_t)g.batch * kMhaHeads * ctx_pad < (1ll << 31);
}

dsa_status_t launch_up_proj(const void* kv_cache, const void* w_uk, const void* w_uv,
                            const Geometry& g, void* k_nope, void* k_rope, void* v,
                            int64_t ctx_pad, cudaStream_t stream) {
  static DeviceOnce once;
  const cudaError_t attr_err = once_per_device(once, [] {
    return cudaFuncSetAttribute(mla_up_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kUpSmemBytes);
  });
  if (attr_err != cudaSuccess) return DSA_ERR_CUDA;
  CUtensorMap tm_lat, tm_uk, tm_uv;
  dsa_status_t st = make_tmap_2d(&tm_lat, kv_cache, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kMhaLat,
                                 (uint64_t)g.cache_rows, 64, 64);
  if (st == DSA_OK)
    st = make_tmap_2d(&tm_uk, w_uk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kMhaDc,
                      (uint64_t)kMhaHeads * kMhaDn, 64, kMhaDn);
  if (st == DSA_OK)
    st = make_tmap_2d(&tm_uv, w_uv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kMhaDc,
                      (uint64_t)kMhaHeads * kMhaDv, 64, kMhaDv);
  if (st != DSA_OK) return st;
  UpProjParams p{};
  p.block_table = g.block_table;
  p.seqlens = g.seqlens;
  p.kv = reinterpret_cast<const __nv_bfloat16*>(kv_cache);
  p.k_nope = reinterpret_cast<__nv_bfloat16*>(k_nope);
  p.k_rope = reinterpret_cast<__nv_bfloat16*>(k_rope);
  p.v = reinterpret_cast<__nv_bfloat16*>(v);
  p.ctx_pad = ctx_pad;
  p.batch = g.batch;
  p.max_ctx = g.max_ctx;
  p.q_per_seq = g.q_per_seq;
  p.paged = g.layout == DSA_KV_PAGED;
  p.page_size = g.page_size;
  p.max_pages = g.max_pages;
  p.num_pages = g.num_pages;
  p.key_tiles = (g.max_ctx + kMhaTile - 1) / kMhaTile;
  p.timeout_ns = g_timeout_ns.load();
  const int64_t items = (int64_t)g.batch * p.key_tiles * kMhaHeads;
  const int grid = (int)std::min<int64_t>(items, num_sms());
  mla_up_proj_kernel<<<grid, kUpThreads, kUpSmemBytes, stream>>>(p, tm_lat, tm_uk, tm_uv);
  return cuda_status(cudaGetLastError());
}

dsa_status_t launch_selection_mask(const int32_t* idx, int k, const Geometry& g, int row_begin,
                                   int row_count, uint32_t* mask, int64_t mask_ld,
                                   cudaStream_t stream) {
  const size_t smem = (size_t)mask_ld * 4;
  if (smem > 227 * 1024) return DSA_ERR_UNSUPPORTED_SHAPE;
  static DeviceOnce once;
  const cudaError_t attr_err = once_per_device(once, [] {
    return cudaFuncSetAttribute(selection_mask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                227 * 1024);
  });
  if (attr_err != cudaSuccess) return DSA_ERR_CUDA;
  MaskParams p{idx, g.seqlens, mask, mask_ld, k, g.batch, g.max_ctx, g.q_per_seq, row_begin,
               row_count, g.q_start, g.num_q};
  const int64_t grid = (int64_t)g.batch * row_count;
  if (grid == 0) return DSA_OK;
  selection_mask_kernel<<<(unsigned)grid, kMaskThreads, smem, stream>>>(p);
  return cuda_status(cudaGetLastError());
}

dsa_status_t launch_masked_mha(const void* q_mha, const void* k_nope, const void* k_rope,
                               const void* v, int64_t ctx_pad, const Geometry& g,
                               const uint32_t* mask, int64_t mask_ld, int k, float scale,
                               void* out, float* lse, cudaStream_t stream) {
  static DeviceOnce once;
  const cudaError_t attr_err = once_per_device(once, [] {
    return cudaFuncSetAttribute(masked_mha_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kFaSmemBytes);
  });
  if (attr_err != cudaSuccess) return DSA_ERR_CUDA;
  CUtensorMap tm_q, tm_kn, tm_kr, tm_v;
  const uint64_t kv_rows = (uint64_t)g.batch * kMhaHeads * ctx_pad;
  dsa_status_t st = make_tmap_3d(&tm_q, q_mha, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kMhaDqk,
                                 kMhaHeads, (uint64_t)g.num_q, 64, 1, kMhaTile);
  if (st == DSA_OK)
    st = make_tmap_2d(&tm_kn, k_nope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kMhaDn, kv_rows, 64,
                      kMhaTile);
  if (st == DSA_OK)
    st = make_tmap_2d(&tm_kr, k_rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kMhaDr,
                      (uint64_t)g.batch * ctx_pad, 64, kMhaTile);
  if (st == DSA_OK)
    st = make_tmap_2d(&tm_v, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kMhaDv, kv_rows, 64,
                      kMhaTile);
  if (st != DSA_OK) return st;
  MhaParams p{};
  p.seqlens = g.seqlens;
  p.mask = mask;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.ctx_pad = ctx_pad;
  p.mask_ld = mask_ld;
  p.batch = g.batch;
  p.max_ctx = g.max_ctx;
  p.q_per_seq = g.q_per_seq;
  p.row_begin = g.row_begin;
  p.row_count = g.row_count;
  p.row_blocks = (g.row_count + kMhaTile - 1) / kMhaTile;
  p.k = k;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load();
  p.q_start = g.q_start;
  p.num_q = g.num_q;
  const int64_t grid = (int64_t)p.row_blocks * g.batch * kMhaHeads;
  if (grid == 0) return DSA_OK;
  masked_mha_kernel<<<(unsigned)grid, kFaThreads, kFaSmemBytes, stream>>>(p, tm_q, tm_kn, tm_kr,
                                                                           tm_v);
  return cuda_status(cudaGetLastError());
}

// ---- fused indexer -> top-k (score rows never stored) ------------------------------------
constexpr int kFuseStride = 8;  // the threshold pass scores every 8th key tile

dsa_status_t launch_cand_select(const Geometry& g, int row_begin, int row_count, int k,
                                int32_t* idx, const uint32_t* ckey, const int32_t* cpos,
                                const uint32_t* cnt, int cap, int32_t* redo_rows,
                                uint32_t* redo_cnt, cudaStream_t stream) {
  static DeviceOnce once;
  const cudaError_t attr_err = once_per_device(once, [] {
    return cudaFuncSetAttribute(cand_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kCandSmemBytes);
  });
  if (attr_err != cudaSuccess) return DSA_ERR_CUDA;
  CandParams p{ckey, cpos, cnt, cap, g.seqlens, g.max_ctx, g.q_per_seq, row_begin, row_count,
               g.batch, k, idx, redo_rows, redo_cnt, g.q_start, g.num_q};
  const int64_t grid = (int64_t)g.batch * row_count;
  if (grid == 0) return DSA_OK;
  cand_select_kernel<<<(unsigned)grid, kCandThreads, kCandSmemBytes, stream>>>(p);
  return cuda_status(cudaGetLastError());
}

struct FusedPlan {
  int64_t ld;           // full score row stride (fallback rows)
  int64_t ld_s;         // sampled score row stride
  int cap;              // candidates kept per row
  int m;                // rank of the threshold within a row's sample
  int chunk_rows;       // window rows per sequence per chunk
  size_t idx_bytes, fallback_bytes, row_bytes;  // row_bytes: per window row of a chunk
};

FusedPlan plan_fused(const Geometry& g, int k, bool need_idx, int cap) {
  FusedPlan f;
  f.ld = (int64_t)(g.max_ctx + kIdxTile - 1) / kIdxTile * kIdxTile;
  const int64_t tiles = f.ld / kIdxTile;
  f.ld_s = ((tiles + kFuseStride - 1) / kFuseStride) * kIdxTile;
  f.cap = cap > 0 ? cap : kCandCap;
  // the k / S largest of a row's sample are expected above its k-th score; the
  // threshold sits 6 standard deviations (and 32) lower, so about 8 (k/S + ...)
  // keys pass per row and fewer than k only far out in the tail (those rows, and
  // rows with more than `cap`, take the full path)
  const int ks = (k + kFuseStride - 1) / kFuseStride;
  f.m = ks + 6 * (int)std::ceil(std::sqrt((double)ks)) + 32;
  f.idx_bytes = need_idx ? align256((size_t)g.num_q * k * 4) : 0;
  f.fallback_bytes = align256((size_t)g.batch * f.ld * 4);
  f.row_bytes = (size_t)f.ld_s * 4 + 4 /*thr*/ + 4 /*cnt*/ + (size_t)f.cap * 8 + 4 /*redo*/;
  int64_t rows = std::max<int64_t>(1, kScoreBudgetBytes / ((int64_t)f.row_bytes * g.batch));
  f.chunk_rows = (int)std::min<int64_t>(rows, g.row_count);
  if (f.chunk_rows >= 4 && f.chunk_rows < g.row_count) f.chunk_rows &= ~3;
  return f;
}

// One chunk of window rows through the fused path; `ws` holds the chunk's buffers.
dsa_status_t select_fused_chunk(const void* q_idx, const float* w, const void* k_idx,
                                const float* k_scale, const Geometry& g, const FusedPlan& f,
                                int k, int r0, int rc, uint8_t* ws, float* fb_scores,
                                int32_t* idx, cudaStream_t s) {
  const int64_t nrow = (int64_t)g.batch * rc;
  float* samp = reinterpret_cast<float*>(ws);
  ws += align256((size_t)nrow * f.ld_s * 4);
  float* thr = reinterpret_cast<float*>(ws);
  ws += align256((size_t)nrow * 4);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(ws);
  ws += align256((size_t)nrow * 4 + 4);  // + the redo counter
  uint32_t* redo_cnt = cnt + nrow;
  int32_t* redo_rows = reinterpret_cast<int32_t*>(ws);
  ws += align256((size_t)nrow * 4);
  uint32_t* ckey = reinterpret_cast<uint32_t*>(ws);
  ws += align256((size_t)nrow * f.cap * 4);
  int32_t* cpos = reinterpret_cast<int32_t*>(ws);
  if (cudaMemsetAsync(cnt, 0, (size_t)(nrow + 1) * 4, s) != cudaSuccess) return DSA_ERR_CUDA;
  // 1. thresholds: the m-th largest score of a strided sample of each row's keys
  dsa_status_t st = launch_indexer(q_idx, w, k_idx, k_scale, g, samp, f.ld_s, r0, rc, s,
                                   kFuseStride);
  if (st == DSA_OK) st = launch_topk(samp, f.ld_s, g, r0, rc, f.m, nullptr, s, kFuseStride, thr);
  // 2. all keys again, keeping only those at or above the row's threshold
  IdxFilter filt;
  filt.thr = thr;
  filt.cand_key = ckey;
  filt.cand_pos = cpos;
  filt.cand_cnt = cnt;
  filt.cand_cap = f.cap;
  if (st == DSA_OK) st = launch_indexer(q_idx, w, k_idx, k_scale, g, samp, f.ld_s, r0, rc, s, 1, filt);
  // 3. the exact top-k of each row's candidates
  if (st == DSA_OK)
    st = launch_cand_select(g, r0, rc, k, idx, ckey, cpos, cnt, f.cap, redo_rows, redo_cnt, s);
  if (st != DSA_OK) return st;
  // 4. rows whose candidates cannot be exact (fewer than k, or more than the list
  //    holds) are selected from their full score rows
  uint32_t n_redo = 0;
  if (cudaMemcpyAsync(&n_redo, redo_cnt, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (n_redo == 0) return DSA_OK;
  n_redo = std::min<uint32_t>(n_redo, (uint32_t)nrow);  // the kernel never lists more
  std::vector<int32_t> rows(n_redo);
  if (cudaMemcpyAsync(rows.data(), redo_rows, (size_t)n_redo * 4, cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DSA_ERR_CUDA;
  std::vector<char> done(rc, 0);  // a window row index covers that row of every sequence
  for (int32_t wr : rows) {
    const int ii = wr % rc;
    if (done[ii]) continue;
    done[ii] = 1;
    st = launch_indexer(q_idx, w, k_idx, k_scale, g, fb_scores, f.ld, r0 + ii, 1, s);
    if (st == DSA_OK) st = launch_topk(fb_scores, f.ld, g, r0 + ii, 1, k, idx, s);
    if (st != DSA_OK) return st;
  }
  return DSA_OK;
}

// ---- scratch for the allocation-free forward ------------------------------------------
// A fixed device array that every device loading this library holds until exit.
// Host code must not use the symbol's host-side address: the device address is
// resolved with cudaGetSymbolAddress, once per device, with that device current.
constexpr size_t kStaticScratchBytes = size_t(128) << 20;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

dsa_status_t static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DSA_OK;
}

// ---- wait-timeout self test ---------------------------------------------------------
__global__ void wait_timeout_selftest_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
  }
  __syncthreads();
  // nothing ever arrives on `bar`: the bounded wait must give up and report
  mbar_wait(smem_u32(&bar), 0, timeout_ns, &abort_flag);
}

}  // namespace

extern "C" {

dsa_status_t dsa_sparse_mla_fwd(const void* q, const void* kv_cache, const dsa_kv_desc_t* kv,
                                const dsa_q_desc_t* qd, const int32_t* idx, int32_t k,
                                float scale, void* out, float* lse, dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, qd, &g);
  if (st != DSA_OK) return st;
  if (!q || !kv_cache || !idx || !out || !lse) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv_cache) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!(scale > 0.f) || !(scale < 1e30f)) return DSA_ERR_INVALID_ARG;
  return launch_sparse_mla(q, kv_cache, g, idx, k, scale, out, lse, (cudaStream_t)stream);
}

dsa_status_t dsa_sparse_mla_fwd_ws(const void* q, const void* kv_cache, const dsa_kv_desc_t* kv,
                                   const dsa_q_desc_t* qd, const int32_t* idx, int32_t k,
                                   float scale, void* workspace, size_t workspace_bytes,
                                   void* out, float* lse, dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, qd, &g);
  if (st != DSA_OK) return st;
  if (!q || !kv_cache || !idx || !out || !lse) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv_cache) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!(scale > 0.f) || !(scale < 1e30f)) return DSA_ERR_INVALID_ARG;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
  return launch_sparse_mla(q, kv_cache, g, idx, k, scale, out, lse, (cudaStream_t)stream,
                           workspace, workspace ? workspace_bytes : 0);
}

size_t dsa_sparse_mla_workspace_size(void) { return (size_t)(num_sms() / 2) * kMlaPartBytes; }

size_t dsa_workspace_size(const dsa_kv_desc_t* kv, const dsa_q_desc_t* q, int32_t k) {
  Geometry g;
  if (check_geometry(kv, q, &g) != DSA_OK || k < 1 || k > kMaxK) return 0;
  const ForwardPlan f = plan_forward(g, k, true);
  // the split top-k's candidates follow a chunk's score rows
  const size_t split = kForwardSplitTopk && split_topk_applies(g, k)
                           ? split_topk_bytes((int64_t)f.chunk_rows * g.batch) : 0;
  // after the selection the score space holds the sparse MLA's split rows
  const MlaSplit sp = plan_mla_split((int64_t)g.batch * g.row_count, k, SIZE_MAX);
  const size_t part_bytes = (size_t)(sp.n_split * sp.nseg) * kMlaPartBytes;
  return f.idx_bytes + std::max(f.score_bytes + split, align256(part_bytes));
}

dsa_status_t dsa_forward(const void* q_idx, const float* w, const void* k_idx,
                         const float* k_scale, const void* q, const void* kv_cache,
                         const dsa_kv_desc_t* kv, const dsa_q_desc_t* qd, int32_t k,
                         float scale, void* workspace, size_t workspace_bytes,
                         int32_t* idx_out, void* out, float* lse, dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, qd, &g);
  if (st != DSA_OK) return st;
  if (!q_idx || !w || !k_idx || !k_scale || !q || !kv_cache || !out || !lse)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(q) || !aligned16(kv_cache) ||
      !aligned16(out))
    return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!(scale > 0.f) || !(scale < 1e30f)) return DSA_ERR_INVALID_ARG;
  ForwardPlan f = plan_forward(g, k, idx_out == nullptr);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < f.idx_bytes)
    return DSA_ERR_WORKSPACE;
  // Long rows take the split top-k when its candidate scratch fits after the score
  // rows. A smaller workspace than dsa_workspace_size() is accepted: the score rows
  // are then processed in smaller chunks (down to one row per sequence), with the
  // split top-k while its scratch still fits beside them, else without it.
  const int64_t row_bytes = f.ld * 4 * g.batch;
  const size_t avail = workspace_bytes - f.idx_bytes;
  bool split = kForwardSplitTopk && split_topk_applies(g, k);
  if (split && avail < f.score_bytes + split_topk_bytes((int64_t)f.chunk_rows * g.batch)) {
    const int64_t per_row = row_bytes + (int64_t)g.batch * (kCandCap * 8 + 4);
    int64_t rows = std::min<int64_t>(f.chunk_rows, ((int64_t)avail - 1024) / per_row);
    if (rows >= 4) rows &= ~int64_t(3);
    if (rows >= 1) {
      f.chunk_rows = (int)rows;
      f.score_bytes = align256((size_t)rows * row_bytes);
    } else {
      split = false;
    }
  }
  if (!split && avail < f.score_bytes) {
    int64_t rows = (int64_t)avail / row_bytes;
    if (rows < 1) return DSA_ERR_WORKSPACE;
    if (rows >= 4) rows &= ~int64_t(3);
    f.chunk_rows = (int)rows;
  }
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws);
  float* scores = reinterpret_cast<float*>(ws + f.idx_bytes);
  void* split_ws = ws + f.idx_bytes + f.score_bytes;
  cudaStream_t s = (cudaStream_t)stream;
  const int r_end = g.row_begin + g.row_count;
  for (int r0 = g.row_begin; r0 < r_end; r0 += f.chunk_rows) {
    const int rc = std::min(f.chunk_rows, r_end - r0);
    st = launch_indexer(q_idx, w, k_idx, k_scale, g, scores, f.ld, r0, rc, s);
    if (st != DSA_OK) return st;
    st = split ? launch_topk_split(scores, f.ld, g, r0, rc, k, idx, s, split_ws)
               : launch_topk(scores, f.ld, g, r0, rc, k, idx, s);
    if (st != DSA_OK) return st;
  }
  // the score rows are dead once the last top-k has run (stream order): their
  // space holds the partial outputs of split rows
  return launch_sparse_mla(q, kv_cache, g, idx, k, scale, out, lse, s, scores,
                           workspace_bytes - f.idx_bytes);
}

dsa_status_t dsa_forward_noalloc(const void* q_idx, const float* w, const void* k_idx,
                                 const float* k_scale, const void* q, const void* kv_cache,
                                 const dsa_kv_desc_t* kv, const dsa_q_desc_t* qd, int32_t k,
                                 float scale, int32_t* idx_out, void* out, float* lse,
                                 dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, qd, &g);
  if (st != DSA_OK) return st;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED_SHAPE;
  // The smallest workspace dsa_forward accepts: the indices (unless the caller
  // receives them in idx_out) plus one score row per sequence.
  const ForwardPlan f = plan_forward(g, k, idx_out == nullptr);
  const size_t min_bytes = f.idx_bytes + align256((size_t)f.ld * 4 * g.batch);
  if (min_bytes > kStaticScratchBytes) return DSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = static_scratch_address(&scratch);
  if (st != DSA_OK) return st;
  return dsa_forward(q_idx, w, k_idx, k_scale, q, kv_cache, kv, qd, k, scale, scratch,
                     kStaticScratchBytes, idx_out, out, lse, stream);
}

dsa_status_t dsa_indexer_kl(const void* q, const void* kv_cache, const dsa_kv_desc_t* kv,
                            const dsa_q_desc_t* qd, const int32_t* idx, int32_t k, float scale,
                            const float* lse, const float* scores, int64_t ld, float* kl,
                            dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, qd, &g);
  if (st != DSA_OK) return st;
  if (!q || !kv_cache || !idx || !lse || !scores || !kl) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv_cache)) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > (1 << 20)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (ld < g.max_ctx) return DSA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !(scale < 1e30f)) return DSA_ERR_INVALID_ARG;
  return launch_indexer_kl(q, kv_cache, g, idx, k, scale, lse, scores, ld, kl,
                           (cudaStream_t)stream);
}

dsa_status_t dsa_mla_up_project(const void* kv_cache, const void* w_uk, const void* w_uv,
                                const dsa_kv_desc_t* kv, void* k_nope, void* k_rope, void* v,
                                int64_t ctx_pad, dsa_stream_t stream) {
  dsa_q_desc_t qd{kv ? kv->batch : 0, 1, 0, 0, nullptr};  // keys only: one nominal row each
  Geometry g;
  dsa_status_t st = check_geometry(kv, &qd, &g);
  if (st != DSA_OK) return st;
  if (!kv_cache || !w_uk || !w_uv || !k_nope || !k_rope || !v) return DSA_ERR_INVALID_ARG;
  if (!aligned16(kv_cache) || !aligned16(w_uk) || !aligned16(w_uv) || !aligned16(k_nope) ||
      !aligned16(k_rope) || !aligned16(v))
    return DSA_ERR_INVALID_ARG;
  const MhaPlan m = plan_mha(g);
  if (ctx_pad < m.ctx_pad || ctx_pad % kMhaTile != 0) return DSA_ERR_INVALID_ARG;
  if (!mha_fits(g, ctx_pad)) return DSA_ERR_UNSUPPORTED_SHAPE;
  return launch_up_proj(kv_cache, w_uk, w_uv, g, k_nope, k_rope, v, ctx_pad,
                        (cudaStream_t)stream);
}

dsa_status_t dsa_selection_mask(const int32_t* idx, int32_t k, const dsa_kv_desc_t* kv,
                                const dsa_q_desc_t* qd, uint32_t* mask, int64_t mask_ld,
                                dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, qd, &g);
  if (st != DSA_OK) return st;
  if (!idx || !mask || !aligned16(mask)) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (mask_ld < plan_mha(g).mask_ld || mask_ld % 4 != 0) return DSA_ERR_INVALID_ARG;
  return launch_selection_mask(idx, k, g, g.row_begin, g.row_count, mask, mask_ld,
                               (cudaStream_t)stream);
}

dsa_status_t dsa_masked_mha(const void* q_mha, const void* k_nope, const void* k_rope,
                            const void* v, int64_t ctx_pad, const dsa_kv_desc_t* kv,
                            const dsa_q_desc_t* qd, const uint32_t* mask, int64_t mask_ld,
                            int32_t k, float scale, void* out, float* lse, dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, qd, &g);
  if (st != DSA_OK) return st;
  if (!q_mha || !k_nope || !k_rope || !v || !out || !lse) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_mha) || !aligned16(k_nope) || !aligned16(k_rope) || !aligned16(v) ||
      !aligned16(out))
    return DSA_ERR_INVALID_ARG;
  const MhaPlan m = plan_mha(g);
  if (ctx_pad < m.ctx_pad || ctx_pad % kMhaTile != 0) return DSA_ERR_INVALID_ARG;
  if (!mha_fits(g, ctx_pad)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (mask) {
    if (!aligned16(mask) || mask_ld < m.mask_ld || mask_ld % 4 != 0) return DSA_ERR_INVALID_ARG;
    if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED_SHAPE;
  }
  if (!(scale > 0.f) || !(scale < 1e30f)) return DSA_ERR_INVALID_ARG;
  return launch_masked_mha(q_mha, k_nope, k_rope, v, ctx_pad, g, mask, mask_ld, mask ? k : 0,
                           scale, out, lse, (cudaStream_t)stream);
}

size_t dsa_mha_workspace_size(const dsa_kv_desc_t* kv, const dsa_q_desc_t* q, int32_t k) {
  Geometry g;
  if (check_geometry(kv, q, &g) != DSA_OK || k < 1 || k > kMaxK) return 0;
  const ForwardPlan f = plan_forward(g, k, true);
  const MhaPlan m = plan_mha(g);
  return f.idx_bytes + f.score_bytes + m.mask_bytes + m.kn_bytes + m.kr_bytes + m.v_bytes;
}

dsa_status_t dsa_mha_prefill(const void* q_idx, const float* w, const void* k_idx,
                             const float* k_scale, const void* q_mha, const void* kv_cache,
                             const void* w_uk, const void* w_uv, const dsa_kv_desc_t* kv,
                             const dsa_q_desc_t* qd, int32_t k, float scale, void* workspace,
                             size_t workspace_bytes, int32_t* idx_out, void* out, float* lse,
                             dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, qd, &g);
  if (st != DSA_OK) return st;
  if (!q_idx || !w || !k_idx || !k_scale || !q_mha || !kv_cache || !w_uk || !w_uv || !out ||
      !lse)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(q_mha) || !aligned16(kv_cache) ||
      !aligned16(w_uk) || !aligned16(w_uv) || !aligned16(out))
    return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!(scale > 0.f) || !(scale < 1e30f)) return DSA_ERR_INVALID_ARG;
  ForwardPlan f = plan_forward(g, k, idx_out == nullptr);
  const MhaPlan m = plan_mha(g);
  if (!mha_fits(g, m.ctx_pad)) return DSA_ERR_UNSUPPORTED_SHAPE;
  const size_t fixed = f.idx_bytes + m.mask_bytes + m.kn_bytes + m.kr_bytes + m.v_bytes;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < fixed)
    return DSA_ERR_WORKSPACE;
  // Rows that select every visible key (pos + 1 <= k) need no scores. Without a
  // seqlens array their positions are known here, so the indexer skips them.
  const int r_end = g.row_begin + g.row_count;
  int sel_begin = g.row_begin;
  if (!g.seqlens && !g.q_start)
    sel_begin = std::min(r_end, std::max(g.row_begin, k - g.max_ctx + g.q_per_seq));
  const int sel_rows = r_end - sel_begin;
  if (sel_rows > 0) {
    const int64_t row_bytes = f.ld * 4 * g.batch;
    int64_t rows = std::min<int64_t>(sel_rows, f.chunk_rows);
    if ((int64_t)(workspace_bytes - fixed) < rows * row_bytes) {
      rows = (int64_t)(workspace_bytes - fixed) / row_bytes;
      if (rows < 1) return DSA_ERR_WORKSPACE;
      if (rows >= 4) rows &= ~int64_t(3);
    }
    f.chunk_rows = (int)rows;
  }
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws);
  ws += f.idx_bytes;
  uint32_t* mask = reinterpret_cast<uint32_t*>(ws);
  ws += m.mask_bytes;
  void* k_nope = ws;
  ws += m.kn_bytes;
  void* k_rope = ws;
  ws += m.kr_bytes;
  void* v = ws;
  ws += m.v_bytes;
  float* scores = reinterpret_cast<float*>(ws);
  cudaStream_t s = (cudaStream_t)stream;
  // selection for the rows that need it, then their masks
  if (idx_out && sel_begin > g.row_begin) {  // all-visible rows: no scores are read
    st = launch_topk(scores, f.ld, g, g.row_begin, sel_begin - g.row_begin, k, idx, s);
    if (st != DSA_OK) return st;
  }
  for (int r0 = sel_begin; r0 < r_end; r0 += f.chunk_rows) {
    const int rc = std::min(f.chunk_rows, r_end - r0);
    st = launch_indexer(q_idx, w, k_idx, k_scale, g, scores, f.ld, r0, rc, s);
    if (st != DSA_OK) return st;
    st = launch_topk(scores, f.ld, g, r0, rc, k, idx, s);
    if (st != DSA_OK) return st;
  }
  if (sel_rows > 0) {
    st = launch_selection_mask(idx, k, g, sel_begin, sel_rows, mask, m.mask_ld, s);
    if (st != DSA_OK) return st;
  }
  st = launch_up_proj(kv_cache, w_uk, w_uv, g, k_nope, k_rope, v, m.ctx_pad, s);
  if (st != DSA_OK) return st;
  return launch_masked_mha(q_mha, k_nope, k_rope, v, m.ctx_pad, g, sel_rows > 0 ? mask : nullptr,
                           m.mask_ld, k, scale, out, lse, s);
}

size_t dsa_fused_workspace_size(const dsa_kv_desc_t* kv, const dsa_q_desc_t* q, int32_t k) {
  Geometry g;
  if (check_geometry(kv, q, &g) != DSA_OK || k < 1 || k > kMaxK) return 0;
  const FusedPlan f = plan_fused(g, k, true, 0);
  const size_t sel = f.fallback_bytes + (size_t)f.chunk_rows * g.batch * f.row_bytes + 8 * 256;
  // dsa_forward_fused: after the selection the same space holds the split rows
  const MlaSplit sp = plan_mla_split((int64_t)g.batch * g.row_count, k, SIZE_MAX);
  return f.idx_bytes + std::max(sel, align256((size_t)(sp.n_split * sp.nseg) * kMlaPartBytes));
}

dsa_status_t dsa_select_fused(const void* q_idx, const float* w, const void* k_idx,
                              const float* k_scale, const dsa_kv_desc_t* kv,
                              const dsa_q_desc_t* qd, int32_t k, int32_t cand_cap,
                              void* workspace, size_t workspace_bytes, int32_t* idx,
                              dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, qd, &g);
  if (st != DSA_OK) return st;
  if (!q_idx || !w || !k_idx || !k_scale || !idx) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx)) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (cand_cap < 0 || cand_cap > kCandCap) return DSA_ERR_INVALID_ARG;
  if ((g.max_ctx + 31) / 32 > kCandMaxWords) return DSA_ERR_UNSUPPORTED_SHAPE;
  FusedPlan f = plan_fused(g, k, false, cand_cap);
  const size_t fixed = f.fallback_bytes + 8 * 256;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < fixed)
    return DSA_ERR_WORKSPACE;
  const int64_t fit = (int64_t)(workspace_bytes - fixed) / ((int64_t)f.row_bytes * g.batch);
  if (fit < 1) return DSA_ERR_WORKSPACE;
  f.chunk_rows = (int)std::min<int64_t>(fit, g.row_count);
  if (f.chunk_rows >= 4 && f.chunk_rows < g.row_count) f.chunk_rows &= ~3;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  float* fb_scores = reinterpret_cast<float*>(ws);
  ws += f.fallback_bytes;
  cudaStream_t s = (cudaStream_t)stream;
  const int r_end = g.row_begin + g.row_count;
  for (int r0 = g.row_begin; r0 < r_end; r0 += f.chunk_rows) {
    const int rc = std::min(f.chunk_rows, r_end - r0);
    st = select_fused_chunk(q_idx, w, k_idx, k_scale, g, f, k, r0, rc, ws, fb_scores, idx, s);
    if (st != DSA_OK) return st;
  }
  return DSA_OK;
}

dsa_status_t dsa_forward_fused(const void* q_idx, const float* w, const void* k_idx,
                               const float* k_scale, const void* q, const void* kv_cache,
                               const dsa_kv_desc_t* kv, const dsa_q_desc_t* qd, int32_t k,
                               float scale, int32_t cand_cap, void* workspace,
                               size_t workspace_bytes, int32_t* idx_out, void* out, float* lse,
                               dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, qd, &g);
  if (st != DSA_OK) return st;
  if (!q || !kv_cache || !out || !lse) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv_cache) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (!(scale > 0.f) || !(scale < 1e30f)) return DSA_ERR_INVALID_ARG;
  const size_t idx_bytes = idx_out ? 0 : align256((size_t)g.num_q * k * 4);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < idx_bytes)
    return DSA_ERR_WORKSPACE;
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(workspace);
  st = dsa_select_fused(q_idx, w, k_idx, k_scale, kv, qd, k, cand_cap,
                        reinterpret_cast<uint8_t*>(workspace) + idx_bytes,
                        workspace_bytes - idx_bytes, idx, stream);
  if (st != DSA_OK) return st;
  // the selection's workspace is dead now: it holds the split rows' partial outputs
  return launch_sparse_mla(q, kv_cache, g, idx, k, scale, out, lse, (cudaStream_t)stream,
                           reinterpret_cast<uint8_t*>(workspace) + idx_bytes,
                           workspace_bytes - idx_bytes);
}

dsa_status_t dsa_selftest_wait_timeout(dsa_stream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(g_timeout_ns.load());
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  return dsa_get_device_error(stream);
}

dsa_status_t dsa_indexer_scores(const void* q_idx, const float* w, const void* k_idx,
                                const float* k_scale, const dsa_kv_desc_t* kv,
                                const dsa_q_desc_t* q, float* scores, int64_t ld,
                                dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, q, &g);
  if (st != DSA_OK) return st;
  if (!q_idx || !w || !k_idx || !k_scale || !scores) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  if (ld < (int64_t)(g.max_ctx + kIdxTile - 1) / kIdxTile * kIdxTile || ld % 4 != 0)
    return DSA_ERR_INVALID_ARG;
  return launch_indexer(q_idx, w, k_idx, k_scale, g, scores, ld, g.row_begin, g.row_count,
                        (cudaStream_t)stream);
}


const char* dsa_status_string(dsa_status_t s) {
  switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG: null pointer, bad size or alignment";
    case DSA_ERR_UNSUPPORTED_SHAPE: return "DSA_ERR_UNSUPPORTED_SHAPE: dims other than the compiled ones";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA: a CUDA runtime call failed";
    case DSA_ERR_DEVICE_TIMEOUT: return "DSA_ERR_DEVICE_TIMEOUT: a bounded device wait ran out";
    case DSA_ERR_BOUNDS: return "DSA_ERR_BOUNDS: an index, page or length was out of range";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE: workspace missing or too small";
  }
  return "unknown dsa_status_t";
}

uint64_t dsa_set_wait_timeout_ns(uint64_t ns) {
  return g_timeout_ns.exchange(ns ? ns : 2000000000ull);
}

dsa_status_t dsa_get_device_error(dsa_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_error_word, sizeof(int));
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  if (word != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int));
    if (e != cudaSuccess) return DSA_ERR_CUDA;
  }
  return (dsa_status_t)word;
}

size_t dsa_topk_workspace_size(const dsa_kv_desc_t* kv, const dsa_q_desc_t* q, int32_t k) {
  Geometry g;
  if (check_geometry(kv, q, &g) != DSA_OK || k < 1 || k > kMaxK) return 0;
  return split_topk_applies(g, k) ? split_topk_bytes((int64_t)g.batch * g.row_count) : 0;
}

dsa_status_t dsa_topk_ws(const float* scores, int64_t ld, const dsa_kv_desc_t* kv,
                         const dsa_q_desc_t* q, int32_t k, void* workspace,
                         size_t workspace_bytes, int32_t* idx, dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, q, &g);
  if (st != DSA_OK) return st;
  if (!scores || !idx) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (ld < g.max_ctx || ld % 4 != 0 || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
  const int64_t rows = (int64_t)g.batch * g.row_count;
  if (workspace && split_topk_applies(g, k) && workspace_bytes >= split_topk_bytes(rows))
    return launch_topk_split(scores, ld, g, g.row_begin, g.row_count, k, idx,
                             (cudaStream_t)stream, workspace);
  return launch_topk(scores, ld, g, g.row_begin, g.row_count, k, idx, (cudaStream_t)stream);
}

dsa_status_t dsa_topk(const float* scores, int64_t ld, const dsa_kv_desc_t* kv,
                      const dsa_q_desc_t* q, int32_t k, int32_t* idx, dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, q, &g);
  if (st != DSA_OK) return st;
  if (!scores || !idx) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (ld < g.max_ctx || ld % 4 != 0 || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  return launch_topk(scores, ld, g, g.row_begin, g.row_count, k, idx, (cudaStream_t)stream);
}

}  // extern "C"

