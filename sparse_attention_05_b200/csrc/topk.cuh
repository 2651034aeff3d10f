// topk.cuh -- fine-grained token selection: per query row, the k highest
// lightning-indexer scores among the visible keys (DeepSeek-V3.2-Exp technical
// report, zh translation, §1 "Architecture" and §2.1: S_t = Top-k(I_{t,:})).
//
// One CTA of 512 threads per row, two per SM. Scores are compared through an
// order-preserving 32-bit key (-0.0 maps to +0.0). The exact selection is a
// radix select:
//   find_kth   histograms of key bits [31:21], [20:10], [9:0] restricted to the
//              prefix found so far (one shared-memory atomic per key; grouping
//              equal digits with match.any first measured slower) -> the exact
//              k-th largest key tau and the number r of keys equal to tau that
//              belong to the selection;
//   compact    one ordered sweep: a key > tau is selected, a key == tau is
//              selected while fewer than r equal keys precede it, so equal
//              scores keep the lower position and the output is ascending.
// Long rows (more than 4k keys) first shrink to a candidate list: a fixed
// strided sample of 2048 scores gives a threshold that lies, with a wide
// margin, below the k-th score; one coalesced sweep keeps the keys at or above
// it, and the exact selection runs on the candidates (rows of up to 131072 keys:
// kept in any order and selected through bitmaps over the positions; longer
// rows: kept in position order and compacted in order). The candidates hold the
// k largest keys whenever there are at least k of them, so the result is exact;
// if the sample misjudged (fewer than k candidates, or more than the buffer
// holds) the row falls back to the exact full-row path.
#pragma once

#include "ptx.cuh"
#include "rows.cuh"

namespace dsa {

constexpr int kTopkThreads = 512;                              // two CTAs (rows) per SM
constexpr int kTopkCacheElems = 16 * 1024;                     // 64 KB: short row or candidates
constexpr int kTopkCandCap = kTopkCacheElems / 2;              // candidates: key + position
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkBinsPerThread = 2048 / kTopkThreads;
constexpr int kTopkSample = 2048;
// cache | hist | misc | sample, then the selection bitmaps of a long row (the second
// one starts over the sample, which is dead by then): 4096 + 4096 words
constexpr int kTopkSmemBytes = kTopkCacheElems * 4 + 2048 * 4 + 64 * 4 + 2 * 4096 * 4;

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
  int32_t* idx;           // [batch * q_per_seq][k], or nullptr: no index output
  // Sampled rows (tile_stride S > 1): a row holds only key tiles 0, S, 2S, ... of the
  // visible keys, compacted; its length is (pos / 128 / S + 1) * 128 (the tail of
  // the last tile is -inf where it lies past pos).
  int32_t tile_stride;
  float* kth_out;         // [batch * row_count] or nullptr: the k-th largest score
  const int32_t* q_start; // [batch + 1] ragged query rows, or nullptr (rows.cuh)
  int32_t num_q;
};

// Inverse of score_key (a key back to its fp32 value; +0.0 for a zero).
__device__ __forceinline__ float key_score(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// fp32 -> key with the same order (as values); -0.0 maps to +0.0.
__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the threads of the block (uint32). Two barriers.
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
    uint32_t w = lane < kTopkWarps ? warp_tot[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < kTopkWarps) warp_tot[lane] = wi - w;  // exclusive
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  return warp_tot[warp] + incl - v;
}

// The k-th largest key among elements [0, n) (k <= n) and how many keys equal to
// it belong to the top k. misc: [0..15] warp totals, [33..34] the pass's result.
// Three barriers per pass: after the histogram, after the warps' bin totals, after
// the result. Each thread owns four consecutive bins (walked from the top), reads
// them once per pass and clears them for the next pass, so hist is all zero again
// on return.
// With passes = 2 only key bits [31:10] are resolved: tau is then the k-th largest
// key with its low 10 bits cleared, a lower bound of it (r_eq is not meaningful).
template <class KeyAt>
__device__ void find_kth(int n, uint32_t k, KeyAt key_at, uint32_t* hist, uint32_t* misc,
                         uint32_t& tau, uint32_t& r_eq, int passes = 3) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_iter = (n + kTopkThreads - 1) / kTopkThreads;
  uint32_t prefix = 0, prefix_mask = 0, remaining = k;
  for (int j = tid; j < 2048; j += kTopkThreads) hist[j] = 0;
  __syncthreads();
#pragma unroll 1
  for (int pass = 0; pass < passes; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);  // key bits [31:21] [20:10] [9:0]
    const uint32_t nbins = pass == 2 ? 1024u : 2048u;
    // histogram of the digits of keys matching the prefix, four keys in flight
#pragma unroll 1
    for (int it = 0; it < n_iter; it += 4) {
      uint32_t digit[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = (it + u) * kTopkThreads + tid;
        digit[u] = 0xFFFFFFFFu;
        if (e < n) {
          const uint32_t key = key_at(e, pass);
          if ((key & prefix_mask) == prefix) digit[u] = (key >> shift) & (nbins - 1);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (digit[u] != 0xFFFFFFFFu) atomicAdd(&hist[digit[u]], 1u);
    }
    __syncthreads();
    // the bin holding the remaining-th largest key: thread tid owns bins
    // 2047 - B tid - i, i < B (B = kTopkBinsPerThread)
    uint32_t cnt[kTopkBinsPerThread], sum = 0;
#pragma unroll
    for (int i = 0; i < kTopkBinsPerThread; ++i) {
      const int bin = 2047 - kTopkBinsPerThread * tid - i;
      cnt[i] = 0u;
      if (bin < (int)nbins) {
        cnt[i] = hist[bin];
        hist[bin] = 0u;
      }
      sum += cnt[i];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) misc[warp] = incl;
    __syncthreads();
    uint32_t above = incl - sum;
    {  // the totals of the warps before this one (four 16-B reads)
      const uint4* t4 = reinterpret_cast<const uint4*>(misc);
#pragma unroll
      for (int q = 0; q < kTopkWarps / 4; ++q) {
        const uint4 t = t4[q];
        above += (4 * q + 0 < warp ? t.x : 0u) + (4 * q + 1 < warp ? t.y : 0u) +
                 (4 * q + 2 < warp ? t.z : 0u) + (4 * q + 3 < warp ? t.w : 0u);
      }
    }
#pragma unroll
    for (int i = 0; i < kTopkBinsPerThread; ++i) {
      if (above < remaining && remaining <= above + cnt[i]) {
        misc[33] = 2047 - kTopkBinsPerThread * tid - i;
        misc[34] = remaining - above;
      }
      above += cnt[i];
    }
    __syncthreads();
    const uint32_t d = misc[33];
    remaining = misc[34];
    prefix |= d << shift;
    prefix_mask |= (nbins - 1) << shift;
  }
  tau = prefix;
  r_eq = remaining;
}

// Ordered compaction of the top k: positions pos_at(e) must increase with e.
template <class KeyAt, class PosAt>
__device__ void compact_topk(int n, uint32_t tau, uint32_t r_eq, KeyAt key_at, PosAt pos_at,
                             int32_t* out, uint32_t* misc) {
  const int tid = threadIdx.x;
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
        keys[u] = key_at(e, 3);
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
        out[gt_b + min(eq_b, r_eq)] = pos_at(e);
        ++gt_b;
      } else if (keys[u] == tau) {
        if (eq_b < r_eq) out[gt_b + eq_b] = pos_at(e);
        ++eq_b;
      }
    }
    gt_run += sweep_tot >> 16;
    eq_run += sweep_tot & 0xFFFFu;
    __syncthreads();  // misc reused by the next sweep's scan
  }
}

// A row of k < n <= 4k <= 8192 keys: staged in shared memory `cache` (all loads in
// flight; rows start 16-B aligned), then the exact top k selected from it. The k-th
// score goes to *kth when kth is given; the selection to out when out is given.
__device__ void select_short_row(const float* row, int n, uint32_t k, float* cache,
                                 uint32_t* hist, uint32_t* misc, int32_t* out, float* kth) {
  const int tid = threadIdx.x;
  {
    constexpr int kPer = 4 * kTopkThreads;
    constexpr int kLoads = 8192 / kPer;  // n <= 4k <= 8192
    float4 v[kLoads];
#pragma unroll
    for (int h = 0; h < kLoads; ++h) {
      const int e0 = h * kPer + 4 * tid;
      if (e0 + 3 < n) {
        v[h] = *reinterpret_cast<const float4*>(row + e0);
      } else {
        v[h].x = e0 < n ? row[e0] : -INFINITY;
        v[h].y = e0 + 1 < n ? row[e0 + 1] : -INFINITY;
        v[h].z = e0 + 2 < n ? row[e0 + 2] : -INFINITY;
        v[h].w = e0 + 3 < n ? row[e0 + 3] : -INFINITY;
      }
    }
#pragma unroll
    for (int h = 0; h < kLoads; ++h) {
      const int e0 = h * kPer + 4 * tid;
      if (e0 < n) *reinterpret_cast<float4*>(cache + e0) = v[h];
    }
    for (int e0 = kLoads * kPer + 4 * tid; e0 < n; e0 += kPer)  // not reached for k <= 2048
      for (int u = 0; u < 4 && e0 + u < n; ++u) cache[e0 + u] = row[e0 + u];
    __syncthreads();
  }
  uint32_t tau, r_eq;
  find_kth(n, k, [&](int e, int) { return score_key(cache[e]); }, hist, misc, tau, r_eq);
  if (kth && tid == 0) *kth = key_score(tau);
  if (out)
    compact_topk(n, tau, r_eq, [&](int e, int) { return score_key(cache[e]); },
                 [&](int e) { return e; }, out, misc);
}

constexpr int kCandThreads = 512;
static_assert(kCandThreads == kTopkThreads, "the shared selection code assumes one block shape");
constexpr int kCandCap = 8192;                     // candidates per row staged in smem
constexpr int kCandMaxWords = 4096;                // bitmap words: rows of <= 131072 keys

// The exact top k of a row of n visible keys from m >= k candidates staged in
// shared memory as (order-preserving key, position) in any order, when they hold
// every key of the row at or above the row's k-th key: the k-th key tau and the
// number r of equal keys to take (find_kth); every key at or above tau marked in a
// bitmap over the row's positions; when more than r keys equal tau, the ones past
// the r lowest positions (an ordered scan of a second bitmap of the equal keys)
// unmarked again; the marks compacted in ascending order into out.
// Bitmaps of (n + 31) / 32 <= kCandMaxWords words; misc[41] counts the equal keys.
// Returns tau; with out == nullptr only tau is found.
__device__ uint32_t select_from_candidates(int m, int n, uint32_t k, const uint32_t* ckey,
                                           const int32_t* cpos, uint32_t* sel, uint32_t* tie,
                                           uint32_t* hist, uint32_t* misc, int32_t* out) {
  const int tid = threadIdx.x;
  const int words = (n + 31) >> 5;
  if (out) {  // ordered before their use by find_kth's first barrier
    for (int w = tid; w < words; w += kTopkThreads) sel[w] = 0u;
    if (tid == 0) misc[41] = 0u;
  }
  uint32_t tau, r_eq;
  find_kth(m, k, [&](int e, int) { return ckey[e]; }, hist, misc, tau, r_eq);
  if (!out) return tau;
  for (int e = tid; e < m; e += kTopkThreads) {
    const uint32_t key = ckey[e];
    if (key >= tau) {
      const int pos = cpos[e];
      atomicOr(&sel[pos >> 5], 1u << (pos & 31));
      if (key == tau) atomicAdd(&misc[41], 1u);
    }
  }
  __syncthreads();
  const int per = (words + kTopkThreads - 1) / kTopkThreads;
  const int w0 = tid * per;
  if (misc[41] > r_eq) {  // block-uniform: ties at tau reach past the selection
    for (int w = tid; w < words; w += kTopkThreads) tie[w] = 0u;
    __syncthreads();
    for (int e = tid; e < m; e += kTopkThreads)
      if (ckey[e] == tau) atomicOr(&tie[cpos[e] >> 5], 1u << (cpos[e] & 31));
    __syncthreads();
    // keep the r_eq lowest positions among the equal keys (each thread owns
    // consecutive words of both bitmaps)
    uint32_t cnt = 0;
    for (int w = w0; w < w0 + per && w < words; ++w) cnt += __popc(tie[w]);
    uint32_t before = block_exclusive_scan(cnt, misc, misc + 32);
    for (int w = w0; w < w0 + per && w < words; ++w) {
      uint32_t bits = tie[w];
      while (bits) {
        const uint32_t bit = bits & (~bits + 1u);
        if (before >= r_eq) sel[w] &= ~bit;
        ++before;
        bits ^= bit;
      }
    }
    __syncthreads();
  }
  // ascending compaction of the selection (exactly k marks)
  uint32_t cnt = 0;
  for (int w = w0; w < w0 + per && w < words; ++w) cnt += __popc(sel[w]);
  uint32_t o = block_exclusive_scan(cnt, misc, misc + 32);
  for (int w = w0; w < w0 + per && w < words; ++w) {
    uint32_t bits = sel[w];
    while (bits) {
      const int bpos = __ffs(bits) - 1;
      if (o < k) out[o] = w * 32 + bpos;
      ++o;
      bits &= bits - 1u;
    }
  }
  return tau;
}

__global__ void __launch_bounds__(kTopkThreads, 2) topk_kernel(TopkParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* cache = reinterpret_cast<float*>(smem_raw);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw + kTopkCacheElems * 4);
  uint32_t* misc = hist + 2048;  // [0..31] warp totals, [32] total, [33..34] results,
                                 // [41] equal keys, [48..63] per-warp kept-key counts
  uint32_t* sample = misc + 64;  // [kTopkSample]
  uint32_t* cand_key = reinterpret_cast<uint32_t*>(cache);      // [kTopkCandCap]
  int32_t* cand_pos = reinterpret_cast<int32_t*>(cache) + kTopkCandCap;
  uint32_t* tie = sample;        // [kCandMaxWords] bitmaps of the long-row selection
  uint32_t* sel = sample + kCandMaxWords;

  const int b = blockIdx.x / p.row_count;
  const int i = p.row_begin + blockIdx.x % p.row_count;
  const SeqRows R = seq_rows(p.q_start, p.seqlens, b, p.q_per_seq, p.num_q, p.max_ctx);
  const int64_t t = R.t0 + i;
  const int tid = threadIdx.x;
  int32_t* out = p.idx && i < R.q_len ? p.idx + t * p.k : nullptr;

  if (!R.ok || i >= R.q_len) {  // a bad sequence, or a window row it does not have
    if (!R.ok && tid == 0) report_error(kErrBounds);
    if (out)
      for (int j = tid; j < p.k; j += kTopkThreads) out[j] = -1;
    if (p.kth_out && tid == 0) p.kth_out[blockIdx.x] = -INFINITY;
    return;
  }
  int n = R.seqlen - R.q_len + i + 1;  // visible keys 0..pos
  if (p.tile_stride > 1) n = ((n - 1) / 128 / p.tile_stride + 1) * 128;  // sampled row
  const uint32_t k = (uint32_t)p.k;
  if (n <= p.k) {
    if (out)
      for (int j = tid; j < p.k; j += kTopkThreads) out[j] = j < n ? j : -1;
    if (p.kth_out && tid == 0) p.kth_out[blockIdx.x] = -INFINITY;
    return;
  }
  const float* row = p.scores + (int64_t)(blockIdx.x) * p.ld;
  uint32_t tau, r_eq;

  if (n > 4 * p.k) {
    // ---- candidate filter ------------------------------------------------------
    // strided sample (a thread's four loads in flight) -> threshold with a wide
    // safety margin below the k-th key
    {
      constexpr int kPer = kTopkSample / kTopkThreads;
      uint32_t sk[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j)
        sk[j] = score_key(row[(int64_t)(tid + j * kTopkThreads) * n / kTopkSample]);
#pragma unroll
      for (int j = 0; j < kPer; ++j) sample[tid + j * kTopkThreads] = sk[j];
    }
    __syncthreads();
    const float frac = (float)p.k / (float)n;
    const float expect = frac * kTopkSample;
    uint32_t r = (uint32_t)(expect + 4.0f * sqrtf(expect) + 16.0f);
    r = min(r, (uint32_t)kTopkSample);
    // two radix passes: the r-th sample key with its low 10 bits cleared, which only
    // lowers the threshold further
    uint32_t tau_low, unused;
    find_kth(kTopkSample, r, [&](int e, int) { return sample[e]; }, hist, misc, tau_low, unused,
             2);
    // key >= tau_low <=> score >= thr (order-preserving keys, -0.0 == +0.0, no NaN)
    const float thr = key_score(tau_low);
    constexpr int kStep = 16 * kTopkThreads;

    if (n <= kCandMaxWords * 32) {
      // Unordered sweep: per step each warp reads 512 consecutive keys (four fully
      // coalesced 16-B pieces per lane) and appends the positions of its kept keys to
      // a region of its own (a warp scan places them; each lane stores one position
      // per kept key), so no step waits on a block barrier or a shared counter. Each
      // lane's pieces arrive by cp.async two steps ahead in one of two 32 KB slots
      // (the candidate keys' and the bitmaps' space, both free until the sweep ends),
      // and each lane reads back only its own pieces, so its cp.async waits are the
      // only synchronisation. Afterwards the regions are packed and the kept keys
      // re-read from the row (in L2 by then). The selection from the candidates works
      // through bitmaps over the row's positions, so their order does not matter.
      // Every warp sees 512 of each 8192 keys, so the regions fill evenly.
      constexpr int kWarpCap = kTopkCandCap / kTopkWarps;  // 512 positions per warp
      const int lane = tid & 31, warp = tid >> 5, wbase = warp * 512 + 4 * lane;
      int32_t* wpos = cand_pos + warp * kWarpCap;
      const uint32_t slot0 = smem_u32(cache), slot1 = smem_u32(tie);
      // this lane's four pieces of the step at `base` into slot `sl` (zero fill past n;
      // those keys are masked)
      auto copy_step = [&](int base, int sl) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e0 = base + wbase + 128 * u;
          const int left = n - e0;
          const uint32_t bytes = left >= 4 ? 16u : (left <= 0 ? 0u : 4u * (uint32_t)left);
          cp_async_16((sl ? slot1 : slot0) + (uint32_t)(wbase + 128 * u) * 4u,
                      bytes ? row + e0 : row, bytes);
        }
        cp_async_commit();
      };
      // The row also streams into L2 a few steps ahead (one thread's bulk prefetches).
      constexpr int kAhead = 4;
      auto prefetch_step = [&](int start) {
        if (tid == 0 && start < n) {
          const int cnt = min(kStep, n - start) & ~3;  // whole 16-B pieces
          if (cnt > 0) prefetch_l2_bulk(row + start, (uint32_t)cnt * 4u);
        }
      };
#pragma unroll
      for (int j = 2; j <= kAhead; ++j) prefetch_step(j * kStep);
      copy_step(0, 0);
      if (kStep < n) copy_step(kStep, 1);
      uint32_t wcount = 0;  // warp-uniform: kept keys this warp has found
#pragma unroll 1
      for (int base = 0, sl = 0; base < n; base += kStep, sl ^= 1) {
        prefetch_step(base + (kAhead + 1) * kStep);
        if (base + kStep < n) cp_async_wait_group<1>();  // this step's pieces have landed
        else cp_async_wait_group<0>();
        float4 cur4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float* src = (sl == 0 ? cache : reinterpret_cast<const float*>(tie)) + wbase + 128 * u;
          cur4[u] = *reinterpret_cast<const float4*>(src);
        }
        uint32_t mask = 0;  // bit 4u + j: key base + wbase + 128u + j is kept
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e0 = base + wbase + 128 * u;
          uint32_t m4 = (cur4[u].x >= thr ? 1u : 0u) | (cur4[u].y >= thr ? 2u : 0u) |
                        (cur4[u].z >= thr ? 4u : 0u) | (cur4[u].w >= thr ? 8u : 0u);
          if (base + kStep > n) {  // the last step: no key at or past n
            const int left = n - e0;
            m4 &= left >= 4 ? 0xFu : (left <= 0 ? 0u : (1u << left) - 1u);
          }
          mask |= m4 << (4 * u);
        }
        // the slot is free again once its values are in registers (the mask above
        // depends on all four reads): the step two ahead goes into it
        if (base + 2 * kStep < n) copy_step(base + 2 * kStep, sl);
        const uint32_t c = __popc(mask);
        uint32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        uint32_t w = wcount + incl - c;
        while (mask) {
          const int bit = __ffs(mask) - 1;
          if (w < (uint32_t)kWarpCap) wpos[w] = base + wbase + 128 * (bit >> 2) + (bit & 3);
          ++w;
          mask &= mask - 1u;
        }
        wcount += __shfl_sync(0xffffffffu, incl, 31);
      }
      cp_async_wait_all();
      if (lane == 0) misc[48 + warp] = wcount;
      __syncthreads();
      uint32_t m = 0, off = 0;
      bool fits = true;
#pragma unroll
      for (int v = 0; v < kTopkWarps; ++v) {
        const uint32_t cv = misc[48 + v];
        fits = fits && cv <= (uint32_t)kWarpCap;
        off += v < warp ? cv : 0u;
        m += cv;
      }
      if (fits && m >= k) {
        // pack the regions (positions held in registers across the barrier) and
        // fetch the keys of the kept positions
        constexpr int kPer = kWarpCap / 32;
        int32_t pos[kPer];
        float x[kPer];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          const uint32_t e = (uint32_t)(lane + 32 * j);
          pos[j] = e < wcount ? wpos[e] : 0;
        }
#pragma unroll
        for (int j = 0; j < kPer; ++j) x[j] = row[pos[j]];
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          const uint32_t e = (uint32_t)(lane + 32 * j);
          if (e < wcount) {
            cand_pos[off + e] = pos[j];
            cand_key[off + e] = score_key(x[j]);
          }
        }
        __syncthreads();  // the packed list, and misc, before the selection
        const uint32_t tau_c =
            select_from_candidates((int)m, n, k, cand_key, cand_pos, sel, tie, hist, misc, out);
        if (p.kth_out && tid == 0) p.kth_out[blockIdx.x] = key_score(tau_c);
        return;
      }
    } else {
      // Rows longer than the bitmaps: keep keys >= tau_low in position order, 16
      // consecutive keys per thread per step (a block scan places them).
      auto load16 = [&](int base, float4 (&v)[4]) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e0 = base + 16 * tid + 4 * u;
          if (e0 + 3 < n) {
            v[u] = *reinterpret_cast<const float4*>(row + e0);
          } else {
            v[u].x = e0 < n ? row[e0] : -INFINITY;
            v[u].y = e0 + 1 < n ? row[e0 + 1] : -INFINITY;
            v[u].z = e0 + 2 < n ? row[e0 + 2] : -INFINITY;
            v[u].w = e0 + 3 < n ? row[e0 + 3] : -INFINITY;
          }
        }
      };
      uint32_t m_run = 0;
      bool overflow = false;
      float4 cur4[4], nxt4[4];
      load16(0, cur4);
#pragma unroll 1
      for (int base = 0; base < n; base += kStep) {
        if (base + kStep < n) load16(base + kStep, nxt4);
        const int e0 = base + 16 * tid;
        uint32_t mask = 0;  // bit u: key e0 + u is kept
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          mask |= (cur4[u].x >= thr ? 1u : 0u) << (4 * u);
          mask |= (cur4[u].y >= thr ? 2u : 0u) << (4 * u);
          mask |= (cur4[u].z >= thr ? 4u : 0u) << (4 * u);
          mask |= (cur4[u].w >= thr ? 8u : 0u) << (4 * u);
        }
        if (base + kStep > n) {  // the last step: no key at or past n
          const int left = n - e0;
          mask &= left >= 16 ? 0xFFFFu : (left <= 0 ? 0u : (1u << left) - 1u);
        }
        const uint32_t excl = block_exclusive_scan(__popc(mask), misc, misc + 32);
        const uint32_t tot = misc[32];
        uint32_t w = m_run + excl;
        if (mask) {
          auto put = [&](int u, float x) {
            if ((mask >> u) & 1u) {
              if (w < (uint32_t)kTopkCandCap) {
                cand_key[w] = score_key(x);
                cand_pos[w] = e0 + u;
              }
              ++w;
            }
          };
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            put(4 * u, cur4[u].x);
            put(4 * u + 1, cur4[u].y);
            put(4 * u + 2, cur4[u].z);
            put(4 * u + 3, cur4[u].w);
          }
        }
        m_run += tot;
        overflow = m_run > (uint32_t)kTopkCandCap;
        __syncthreads();
        if (overflow) break;
#pragma unroll
        for (int u = 0; u < 4; ++u) cur4[u] = nxt4[u];
      }
      if (!overflow && m_run >= k) {
        const int m = (int)m_run;
        find_kth(m, k, [&](int e, int) { return cand_key[e]; }, hist, misc, tau, r_eq);
        if (p.kth_out && tid == 0) p.kth_out[blockIdx.x] = key_score(tau);
        if (out)
          compact_topk(m, tau, r_eq, [&](int e, int) { return cand_key[e]; },
                       [&](int e) { return cand_pos[e]; }, out, misc);
        return;
      }
    }
    // the sample misjudged this row: exact selection over the whole row
    __syncthreads();
    find_kth(n, k, [&](int e, int) { return score_key(row[e]); }, hist, misc, tau, r_eq);
    if (p.kth_out && tid == 0) p.kth_out[blockIdx.x] = key_score(tau);
    if (out)
      compact_topk(n, tau, r_eq, [&](int e, int) { return score_key(row[e]); },
                   [&](int e) { return e; }, out, misc);
    return;
  }

  // ---- short rows: staged in shared memory, then selected ----
  select_short_row(row, n, k, cache, hist, misc, out, p.kth_out ? p.kth_out + blockIdx.x : nullptr);
}

// ======================================================================================
// Selection from a candidate list (the fused indexer -> top-k path)
// ======================================================================================
// Each window row comes with the keys the indexer's filter kept: every visible key
// whose score reached the row's threshold, as (order-preserving key, position) in no
// particular order. When the list holds at least k keys (and all of them: count <=
// capacity), it contains the k largest of the row, so the exact top-k is selected
// from it: the k-th key tau and the number r of equal keys to take (find_kth), keys
// above tau marked in a bitmap over the row's positions, the r lowest positions of
// the keys equal to tau marked from a second bitmap, and the marks compacted in
// ascending order. Other rows are listed for the full (unfused) selection.
struct CandParams {
  const uint32_t* cand_key;  // [batch * row_count][cand_cap]
  const int32_t* cand_pos;   // [batch * row_count][cand_cap]
  const uint32_t* cand_cnt;  // [batch * row_count]
  int32_t cand_cap;          // <= kCandCap
  const int32_t* seqlens;    // [batch] or nullptr
  int32_t max_ctx, q_per_seq, row_begin, row_count, batch, k;
  int32_t* idx;              // [num_q][k]
  int32_t* redo_rows;        // [batch * row_count] window rows left to the full path
  uint32_t* redo_cnt;        // how many (zeroed by the caller)
  const int32_t* q_start;    // [batch + 1] ragged query rows, or nullptr (rows.cuh)
  int32_t num_q;
};

constexpr int kCandSmemBytes =
    kCandCap * 8 + 2 * kCandMaxWords * 4 + 2048 * 4 + 64 * 4;

__global__ void __launch_bounds__(kCandThreads, 2) cand_select_kernel(CandParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* ckey = reinterpret_cast<uint32_t*>(smem_raw);          // [kCandCap]
  int32_t* cpos = reinterpret_cast<int32_t*>(ckey + kCandCap);     // [kCandCap]
  uint32_t* sel = reinterpret_cast<uint32_t*>(cpos + kCandCap);    // [kCandMaxWords]
  uint32_t* tie = sel + kCandMaxWords;                             // [kCandMaxWords]
  uint32_t* hist = tie + kCandMaxWords;                            // [2048]
  uint32_t* misc = hist + 2048;                                    // [64]

  const int64_t wrow = blockIdx.x;
  const int b = (int)(wrow / p.row_count);
  const int i = p.row_begin + (int)(wrow - (int64_t)b * p.row_count);
  const SeqRows R = seq_rows(p.q_start, p.seqlens, b, p.q_per_seq, p.num_q, p.max_ctx);
  const int64_t t = R.t0 + i;
  const int tid = threadIdx.x;
  int32_t* out = i < R.q_len ? p.idx + t * p.k : nullptr;
  if (!R.ok || i >= R.q_len) {  // a bad sequence, or a window row it does not have
    if (!R.ok && tid == 0) report_error(kErrBounds);
    if (out)
      for (int j = tid; j < p.k; j += kCandThreads) out[j] = -1;
    return;
  }
  const int n = R.seqlen - R.q_len + i + 1;  // visible keys 0..pos
  if (n <= p.k) {
    for (int j = tid; j < p.k; j += kCandThreads) out[j] = j < n ? j : -1;
    return;
  }
  const uint32_t m = p.cand_cnt[wrow];
  if (m < (uint32_t)p.k || m > (uint32_t)p.cand_cap) {
    if (tid == 0) {  // one entry per row at most, so the slot stays below the row count
      const uint32_t slot = atomicAdd(p.redo_cnt, 1u);
      if (slot < (uint32_t)p.batch * (uint32_t)p.row_count) p.redo_rows[slot] = (int32_t)wrow;
    }
    return;
  }
  for (uint32_t e = tid; e < m; e += kCandThreads) {
    ckey[e] = p.cand_key[wrow * p.cand_cap + e];
    cpos[e] = p.cand_pos[wrow * p.cand_cap + e];
  }
  select_from_candidates((int)m, n, (uint32_t)p.k, ckey, cpos, sel, tie, hist, misc, out);
}


// ======================================================================================
// Long rows split across CTAs (the unfused selection with a scratch buffer)
// ======================================================================================
// One CTA per row holds a long row's whole sweep: a 131072-key row takes 16 sweep
// steps of 8192 keys one after the other, and with few rows (decode) the longest
// rows alone set the time. Here the sweep of a row with more than 4k keys is cut
// into chunks of kSplitChunk keys, one CTA each (topk_sweep_kernel): each chunk CTA
// takes the row threshold (computed once per row by topk_threshold_kernel from the
// same strided sample of 2048 scores as the one-CTA path) and appends the keys of its
// chunk at or above it to the row's candidate list with one atomic per warp and step
// (no block barrier per step, in no particular order). topk_select_kernel then selects per row: rows of at most 4k
// keys from their scores staged in shared memory, long rows from their candidates
// (select_from_candidates) when there are at least k of them and no more than the
// list holds -- they then hold every key at or above the row's k-th -- and the
// others by the exact full-row path. The result equals topk_kernel's bit for bit.
constexpr int kSplitChunk = 16384;  // keys per sweep CTA (64 KB of scores)

struct SplitParams {
  const float* scores;     // [batch * row_count][ld]
  int64_t ld;
  const int32_t* seqlens;  // [batch] or nullptr
  const int32_t* q_start;  // [batch + 1] ragged query rows, or nullptr (rows.cuh)
  int32_t num_q, max_ctx, q_per_seq, row_begin, row_count, batch, k;
  int32_t nchunk;          // sweep chunks per window row: ceil(max_ctx / kSplitChunk)
  uint32_t* cand_key;      // [batch * row_count][kCandCap]
  int32_t* cand_pos;       // [batch * row_count][kCandCap]
  uint32_t* cand_cnt;      // [batch * row_count], zeroed by topk_threshold_kernel
  uint32_t* thr_key;       // [batch * row_count] long rows' threshold keys
  int32_t* idx;            // [num_q][k] (topk_select_kernel)
};

// Window row `wrow` of the split top-k: its global row t and visible keys n (0 when
// the row does not exist or its sequence is invalid).
__device__ __forceinline__ int split_row(const SplitParams& p, int64_t wrow, int64_t& t,
                                         bool& ok) {
  const int b = (int)(wrow / p.row_count);
  const int i = p.row_begin + (int)(wrow - (int64_t)b * p.row_count);
  const SeqRows R = seq_rows(p.q_start, p.seqlens, b, p.q_per_seq, p.num_q, p.max_ctx);
  t = R.t0 + i;
  ok = R.ok;
  if (!R.ok || i >= R.q_len) return 0;
  return R.seqlen - R.q_len + i + 1;
}

// Threshold key of a long row: the r-th largest of the fixed strided sample of 2048
// scores, r = the expected count of top-k keys in the sample + 4 standard deviations
// + 16 (topk_kernel's one-CTA path takes the same key with its low 10 bits cleared).
// One CTA of 4 warps per row computes it: each thread holds 16 sampled keys, and four
// passes over 8-bit digits (a 256-bin histogram of shared atomics, then a scan of the
// bins by warp 0) narrow the prefix down to the exact key.
constexpr int kThresholdThreads = 128;

__device__ __forceinline__ uint32_t sample_threshold(const float* row, int n, uint32_t k,
                                                     uint32_t* hist, uint32_t* bcast) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kPer = kTopkSample / kThresholdThreads;  // 16 sampled keys per thread
  uint32_t key[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j)
    key[j] = score_key(row[(int64_t)(tid + kThresholdThreads * j) * n / kTopkSample]);
  const float expect = (float)k / (float)n * kTopkSample;
  uint32_t remaining = (uint32_t)(expect + 4.0f * sqrtf(expect) + 16.0f);
  remaining = min(remaining, (uint32_t)kTopkSample);
  uint32_t prefix = 0, mask = 0;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += kThresholdThreads) hist[b] = 0u;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const uint32_t digit = (key[j] & mask) == prefix ? (key[j] >> shift) & 255u : 256u;
      if (digit < 256u) atomicAdd(&hist[digit], 1u);
    }
    __syncthreads();
    if (warp == 0) {  // bins from the top: lane l owns bins 255 - 8 l - i, i < 8
      uint32_t cnt[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = hist[255 - 8 * lane - i];
        sum += cnt[i];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
      }
      uint32_t above = incl - sum;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (above < remaining && remaining <= above + cnt[i]) {  // exactly one (lane, i)
          bcast[0] = 255u - 8u * lane - i;
          bcast[1] = remaining - above;
        }
        above += cnt[i];
      }
    }
    __syncthreads();
    prefix |= bcast[0] << shift;
    mask |= 255u << shift;
    remaining = bcast[1];
  }
  return prefix;
}

// One CTA per window row: zeroes the row's candidate count and, for a long row,
// computes its threshold key once for all of its chunk CTAs.
__global__ void __launch_bounds__(kThresholdThreads) topk_threshold_kernel(SplitParams p) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t bcast[2];
  const int64_t wrow = blockIdx.x;
  int64_t t;
  bool ok;
  const int n = split_row(p, wrow, t, ok);
  if (threadIdx.x == 0) p.cand_cnt[wrow] = 0u;
  if (n <= 4 * p.k) return;
  const uint32_t thr = sample_threshold(p.scores + wrow * p.ld, n, (uint32_t)p.k, hist, bcast);
  if (threadIdx.x == 0) p.thr_key[wrow] = thr;
}

// Sweep of keys [c0, c1) of a long row (c1 - c0 <= kSplitChunk, c0 a multiple of 16):
// 16 consecutive keys per thread per step (8192 keys), both steps' loads issued before
// either is used; keys with a score >= thr (<=> key >= the threshold key: no NaN
// scores) are appended to the row's list. The CTA reserves its slots with one atomic
// for the whole chunk (a block scan of the threads' counts: every chunk CTA of a row
// adds to the same counter, so per-warp atomics would queue at one address); slots
// past kCandCap are counted but not written. `scan` is 32 words of shared memory.
__device__ __forceinline__ void sweep_chunk(const float* row, int c0, int c1, float thr,
                                            uint32_t* cnt, uint32_t* ckey, int32_t* cpos,
                                            uint32_t* scan) {
  constexpr int kStep = 16 * kTopkThreads;
  static_assert(kSplitChunk == 2 * kStep, "two sweep steps per chunk");
  const int tid = threadIdx.x;
  float4 v[2][4];
#pragma unroll
  for (int s = 0; s < 2; ++s)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e0 = c0 + s * kStep + 16 * tid + 4 * u;  // rows and chunks are 16-B aligned
      if (e0 + 3 < c1) {
        v[s][u] = *reinterpret_cast<const float4*>(row + e0);
      } else {
        v[s][u].x = e0 < c1 ? row[e0] : -INFINITY;
        v[s][u].y = e0 + 1 < c1 ? row[e0 + 1] : -INFINITY;
        v[s][u].z = e0 + 2 < c1 ? row[e0 + 2] : -INFINITY;
        v[s][u].w = e0 + 3 < c1 ? row[e0 + 3] : -INFINITY;
      }
    }
  uint32_t mask[2];  // bit j of mask[s]: key c0 + s kStep + 16 tid + j is kept
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    uint32_t m = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      m |= (v[s][u].x >= thr ? 1u : 0u) << (4 * u);
      m |= (v[s][u].y >= thr ? 2u : 0u) << (4 * u);
      m |= (v[s][u].z >= thr ? 4u : 0u) << (4 * u);
      m |= (v[s][u].w >= thr ? 8u : 0u) << (4 * u);
    }
    const int left = c1 - (c0 + s * kStep + 16 * tid);  // -inf past c1 never passes; be exact
    mask[s] = m & (left >= 16 ? 0xFFFFu : (left <= 0 ? 0u : (1u << left) - 1u));
  }
  const uint32_t mine = __popc(mask[0]) + __popc(mask[1]);
  const uint32_t before = block_exclusive_scan(mine, scan, scan + 16);
  if (tid == 0 && scan[16] > 0u) scan[17] = atomicAdd(cnt, scan[16]);
  __syncthreads();
  uint32_t w = scan[17] + before;
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int e0 = c0 + s * kStep + 16 * tid;
    auto put = [&](int j, float x) {
      if ((mask[s] >> j) & 1u) {
        if (w < (uint32_t)kCandCap) {
          ckey[w] = score_key(x);
          cpos[w] = e0 + j;
        }
        ++w;
      }
    };
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      put(4 * u, v[s][u].x);
      put(4 * u + 1, v[s][u].y);
      put(4 * u + 2, v[s][u].z);
      put(4 * u + 3, v[s][u].w);
    }
  }
  __syncthreads();  // scan[] is reused by the CTA's next chunk
}

// One CTA per (row, chunk); a CTA whose row is short or whose chunk lies past the row
// exits at once.
__global__ void __launch_bounds__(kTopkThreads, 1) topk_sweep_kernel(SplitParams p) {
  __shared__ uint32_t scan[32];
  const int64_t wrow = blockIdx.x / p.nchunk;
  const int chunk = (int)(blockIdx.x - wrow * p.nchunk);
  int64_t t;
  bool ok;
  const int n = split_row(p, wrow, t, ok);
  const int c0 = chunk * kSplitChunk;
  if (n <= 4 * p.k || c0 >= n) return;  // short rows and chunks past the row: no sweep
  const int c1 = min(n, c0 + kSplitChunk);
  sweep_chunk(p.scores + wrow * p.ld, c0, c1, key_score(p.thr_key[wrow]), p.cand_cnt + wrow,
              p.cand_key + wrow * kCandCap, p.cand_pos + wrow * kCandCap, scan);
}

constexpr int kSelectSmemBytes =
    kCandCap * 8 + 2 * kCandMaxWords * 4 + 2048 * 4 + 64 * 4;

__global__ void __launch_bounds__(kTopkThreads, 2) topk_select_kernel(SplitParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* ckey = reinterpret_cast<uint32_t*>(smem_raw);          // [kCandCap]
  int32_t* cpos = reinterpret_cast<int32_t*>(ckey + kCandCap);     // [kCandCap]
  float* cache = reinterpret_cast<float*>(smem_raw);               // short rows (<= 8192)
  uint32_t* sel = reinterpret_cast<uint32_t*>(cpos + kCandCap);    // [kCandMaxWords]
  uint32_t* tie = sel + kCandMaxWords;                             // [kCandMaxWords]
  uint32_t* hist = tie + kCandMaxWords;                            // [2048]
  uint32_t* misc = hist + 2048;                                    // [64]
  const int64_t wrow = blockIdx.x;
  const int tid = threadIdx.x;
  int64_t t;
  bool ok;
  const int n = split_row(p, wrow, t, ok);
  if (n == 0) {  // a bad sequence (reported; its existing rows padded), or no such row
    const int b = (int)(wrow / p.row_count);
    const int i = p.row_begin + (int)(wrow - (int64_t)b * p.row_count);
    if (!ok) {
      if (tid == 0) report_error(kErrBounds);
      if (!p.q_start && i < p.q_per_seq)
        for (int j = tid; j < p.k; j += kTopkThreads) p.idx[t * p.k + j] = -1;
    }
    return;
  }
  int32_t* out = p.idx + t * p.k;
  const uint32_t k = (uint32_t)p.k;
  if (n <= p.k) {
    for (int j = tid; j < p.k; j += kTopkThreads) out[j] = j < n ? j : -1;
    return;
  }
  const float* row = p.scores + wrow * p.ld;
  if (n <= 4 * p.k) {
    select_short_row(row, n, k, cache, hist, misc, out, nullptr);
    return;
  }
  const uint32_t m = p.cand_cnt[wrow];
  if (m >= k && m <= (uint32_t)kCandCap) {
    for (uint32_t e = tid; e < m; e += kTopkThreads) {
      ckey[e] = p.cand_key[wrow * kCandCap + e];
      cpos[e] = p.cand_pos[wrow * kCandCap + e];
    }
    select_from_candidates((int)m, n, k, ckey, cpos, sel, tie, hist, misc, out);
    return;
  }
  // the sample misjudged this row: exact selection over the whole row
  uint32_t tau, r_eq;
  find_kth(n, k, [&](int e, int) { return score_key(row[e]); }, hist, misc, tau, r_eq);
  compact_topk(n, tau, r_eq, [&](int e, int) { return score_key(row[e]); },
               [&](int e) { return e; }, out, misc);
}

}  // namespace dsa
