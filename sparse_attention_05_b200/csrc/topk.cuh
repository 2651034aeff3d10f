// topk.cuh -- fine-grained token selection: per query row, the k highest
// lightning-indexer scores among the visible keys (DeepSeek-V3.2-Exp technical
// report, zh translation, §1 "Architecture" and §2.1: S_t = Top-k(I_{t,:})).
//
// One CTA of 1024 threads per row, radix select on an order-preserving 32-bit
// key of each fp32 score:
//   pass 1..3  histograms of key bits [31:21], [20:10], [9:0] restricted to the
//              prefix found so far -> the exact k-th largest key tau and the
//              number r of keys equal to tau that belong to the selection;
//   compaction one ordered sweep: a key > tau is selected, a key == tau is
//              selected while fewer than r equal keys precede it, so equal
//              scores keep the lower position and the output is ascending.
// Rows of up to kTopkCacheElems scores stay in shared memory across passes;
// longer rows are re-read from global memory (L2) on every pass.
#pragma once

#include "ptx.cuh"

namespace dsa {

constexpr int kTopkThreads = 1024;
constexpr int kTopkCacheElems = 40 * 1024;                     // 160 KB row cache
constexpr int kTopkSmemBytes = kTopkCacheElems * 4 + 2048 * 4 + 64 * 4;

struct TopkParams {
  const float* scores;
  int64_t ld;             // row stride of scores (elements)
  const int32_t* seqlens; // [batch] or nullptr
  int32_t max_ctx;
  int32_t q_per_seq;
  int32_t row_begin;      // rows [row_begin, row_begin + row_count) of every sequence
  int32_t row_count;
  int32_t batch;
  int32_t k;
  int32_t* idx;           // [batch * q_per_seq][k]
};

// fp32 -> key with the same order (as values); -0.0 maps to +0.0.
__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the 1024 threads of the block (uint32). Two barriers.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tot,
                                                         uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_tot[lane];
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    warp_tot[lane] = wi - w;  // exclusive
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  return warp_tot[warp] + incl - v;
}

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(TopkParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* cache = reinterpret_cast<float*>(smem_raw);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw + kTopkCacheElems * 4);
  uint32_t* misc = hist + 2048;  // [0..31] warp totals, [32] total, [33] digit, [34] remaining

  const int b = blockIdx.x / p.row_count;
  const int i = p.row_begin + blockIdx.x % p.row_count;
  const int64_t t = (int64_t)b * p.q_per_seq + i;
  const int tid = threadIdx.x;
  int32_t* out = p.idx + t * p.k;

  const int seqlen = p.seqlens ? p.seqlens[b] : p.max_ctx;
  if (seqlen < p.q_per_seq || seqlen > p.max_ctx) {
    if (tid == 0) report_error(kErrBounds);
    for (int j = tid; j < p.k; j += kTopkThreads) out[j] = -1;
    return;
  }
  const int n = seqlen - p.q_per_seq + i + 1;  // visible keys 0..pos
  if (n <= p.k) {
    for (int j = tid; j < p.k; j += kTopkThreads) out[j] = j < n ? j : -1;
    return;
  }

  const float* row = p.scores + (int64_t)(blockIdx.x) * p.ld;
  const bool cached = n <= kTopkCacheElems;
  const int n_iter = (n + kTopkThreads - 1) / kTopkThreads;

  uint32_t prefix = 0;       // key bits fixed so far
  uint32_t prefix_mask = 0;  // which bits of the key are fixed
  uint32_t remaining = p.k;  // how many of the k still lie at or below the prefix

  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const uint32_t nbins = 1u << widths[pass];
    for (int j = tid; j < 2048; j += kTopkThreads) hist[j] = 0;
    __syncthreads();
#pragma unroll 1
    for (int it = 0; it < n_iter; ++it) {
      const int e = it * kTopkThreads + tid;
      uint32_t digit = 0xFFFFFFFFu;
      if (e < n) {
        float x;
        if (pass == 0) {
          x = row[e];
          if (cached) cache[e] = x;
        } else {
          x = cached ? cache[e] : row[e];
        }
        const uint32_t key = score_key(x);
        if ((key & prefix_mask) == prefix) digit = (key >> shift) & (nbins - 1);
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, digit);
      if (digit != 0xFFFFFFFFu && (__ffs(peers) - 1) == (tid & 31))
        atomicAdd(&hist[digit], __popc(peers));
    }
    __syncthreads();
    // Find the bin holding the remaining-th largest key: threads walk the bins
    // from the top, two bins per thread (bins 2047-2*tid and 2046-2*tid).
    const int hi_bin = 2047 - 2 * tid, lo_bin = 2046 - 2 * tid;
    const uint32_t c_hi = hi_bin < (int)nbins ? hist[hi_bin] : 0;
    const uint32_t c_lo = lo_bin < (int)nbins ? hist[lo_bin] : 0;
    const uint32_t above = block_exclusive_scan(c_hi + c_lo, misc, misc + 32);
    if (above < remaining && remaining <= above + c_hi) {
      misc[33] = hi_bin;
      misc[34] = remaining - above;
    } else if (above + c_hi < remaining && remaining <= above + c_hi + c_lo) {
      misc[33] = lo_bin;
      misc[34] = remaining - above - c_hi;
    }
    __syncthreads();
    const uint32_t d = misc[33];
    remaining = misc[34];
    prefix |= d << shift;
    prefix_mask |= (nbins - 1) << shift;
    __syncthreads();
  }
  const uint32_t tau = prefix;      // exact key of the k-th largest score
  const uint32_t r_eq = remaining;  // keys == tau to take, lowest positions first

  // Ordered compaction: each thread owns 8 consecutive positions per sweep.
  uint32_t gt_run = 0, eq_run = 0;  // selected-above / equal counts before this sweep
  const int per_sweep = kTopkThreads * 8;
#pragma unroll 1
  for (int base = 0; base < n; base += per_sweep) {
    const int e0 = base + tid * 8;
    uint32_t keys[8];
    uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + u;
      keys[u] = 0;
      if (e < n) {
        keys[u] = score_key(cached ? cache[e] : row[e]);
        n_gt += keys[u] > tau;
        n_eq += keys[u] == tau;
      }
    }
    // Pack (gt, eq) counts: each at most 8 per thread, 8192 per sweep.
    const uint32_t excl = block_exclusive_scan((n_gt << 16) | n_eq, misc, misc + 32);
    const uint32_t sweep_tot = misc[32];
    uint32_t gt_b = gt_run + (excl >> 16), eq_b = eq_run + (excl & 0xFFFFu);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + u;
      if (e >= n) break;
      if (keys[u] > tau) {
        out[gt_b + min(eq_b, r_eq)] = e;
        ++gt_b;
      } else if (keys[u] == tau) {
        if (eq_b < r_eq) out[gt_b + eq_b] = e;
        ++eq_b;
      }
    }
    gt_run += sweep_tot >> 16;
    eq_run += sweep_tot & 0xFFFFu;
    __syncthreads();  // misc reused by the next sweep's scan
  }
}

}  // namespace dsa
