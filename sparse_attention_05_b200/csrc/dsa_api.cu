// dsa_api.cu -- the C ABI of include/dsa.h: host-side argument checks, launch
// geometry and the dsa_forward orchestration over the three kernels.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/dsa.h"
#include "ptx.cuh"
#include "topk.cuh"
#include "indexer.cuh"
#include "sparse_mla.cuh"

using namespace dsa;

namespace {

constexpr int kHIdx = 64, kDIdx = 128, kHeads = 128, kDqk = 576, kDv = 512, kMaxK = 2048;

std::atomic<uint64_t> g_timeout_ns{2000000000ull};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dsa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

// Validated geometry shared by every entry point.
struct Geometry {
  int layout, batch, max_ctx, page_size, num_pages, max_pages, q_per_seq, num_q;
  const int32_t* block_table;
  const int32_t* seqlens;
  int64_t cache_rows;  // rows of each per-token cache array
};

dsa_status_t check_geometry(const dsa_kv_desc_t* kv, const dsa_q_desc_t* q, Geometry* g) {
  if (!kv || !q) return DSA_ERR_INVALID_ARG;
  if (kv->batch < 1 || kv->max_ctx < 1 || q->q_per_seq < 1) return DSA_ERR_INVALID_ARG;
  if ((int64_t)kv->batch * q->q_per_seq != q->num_q) return DSA_ERR_INVALID_ARG;
  if (q->q_per_seq > kv->max_ctx) return DSA_ERR_INVALID_ARG;
  g->layout = kv->layout;
  g->batch = kv->batch;
  g->max_ctx = kv->max_ctx;
  g->q_per_seq = q->q_per_seq;
  g->num_q = q->num_q;
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

int num_sms() {
  static int sms = [] {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
  }();
  return sms;
}

// ---- top-k launch ------------------------------------------------------------------
dsa_status_t launch_topk(const float* scores, int64_t ld, const Geometry& g, int row_begin,
                         int row_count, int k, int32_t* idx, cudaStream_t stream) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kTopkSmemBytes);
  });
  if (attr_err != cudaSuccess) return DSA_ERR_CUDA;
  TopkParams p{scores, ld, g.seqlens, g.max_ctx, g.q_per_seq, row_begin, row_count, g.batch, k, idx};
  const int64_t grid = (int64_t)g.batch * row_count;
  if (grid == 0) return DSA_OK;
  topk_kernel<<<(unsigned)grid, kTopkThreads, kTopkSmemBytes, stream>>>(p);
  return cuda_status(cudaGetLastError());
}

}  // namespace

extern "C" {

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

dsa_status_t dsa_topk(const float* scores, int64_t ld, const dsa_kv_desc_t* kv,
                      const dsa_q_desc_t* q, int32_t k, int32_t* idx, dsa_stream_t stream) {
  Geometry g;
  dsa_status_t st = check_geometry(kv, q, &g);
  if (st != DSA_OK) return st;
  if (!scores || !idx) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (ld < g.max_ctx) return DSA_ERR_INVALID_ARG;
  return launch_topk(scores, ld, g, 0, g.q_per_seq, k, idx, (cudaStream_t)stream);
}

}  // extern "C"

// TEMPORARY stubs (replaced as the kernels land)
extern "C" {
dsa_status_t dsa_indexer_scores(const void*, const float*, const void*, const float*,
                                const dsa_kv_desc_t*, const dsa_q_desc_t*, float*, int64_t,
                                dsa_stream_t) { return DSA_ERR_UNSUPPORTED_SHAPE; }
dsa_status_t dsa_sparse_mla_fwd(const void*, const void*, const dsa_kv_desc_t*,
                                const dsa_q_desc_t*, const int32_t*, int32_t, float, void*,
                                float*, dsa_stream_t) { return DSA_ERR_UNSUPPORTED_SHAPE; }
size_t dsa_workspace_size(const dsa_kv_desc_t*, const dsa_q_desc_t*, int32_t) { return 0; }
dsa_status_t dsa_forward(const void*, const float*, const void*, const float*, const void*,
                         const void*, const dsa_kv_desc_t*, const dsa_q_desc_t*, int32_t, float,
                         void*, size_t, int32_t*, void*, float*, dsa_stream_t) {
  return DSA_ERR_UNSUPPORTED_SHAPE;
}
dsa_status_t dsa_selftest_wait_timeout(dsa_stream_t) { return DSA_ERR_UNSUPPORTED_SHAPE; }
}
