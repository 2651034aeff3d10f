// indexer.cuh -- lightning indexer scores on the sm_100a tensor cores.
//
// DeepSeek-V3.2-Exp technical report (zh translation), §1 "Architecture", Eq. 1:
//   I_{t,s} = sum_j w_{t,j} * ReLU(q^I_{t,j} . k^I_s),  keys s <= pos(t),
// implemented in FP8 as that section allows: keys arrive as E4M3 codes with one
// fp32 scale s_k per token; each (token, head) query row is quantized here to
// E4M3 with s_q = max(amax, 2^-120) / 448, so that
//   I_{t,s} = s_k[s] * sum_j (w_{t,j} s_q[t,j]) * ReLU(q_hat_{t,j} . k_hat_s).
//
// One persistent CTA per SM. The work is the ordered list of 128-key tiles of
// every (sequence, group of G <= 4 query rows); each CTA computes the total
// from the sequence lengths itself and takes an exact equal share of that list
// (sequences of very different lengths are balanced without any workspace).
// A unit is the run of one group's tiles inside the share. Per key tile the tensor core computes
//   D[key][(row, head)] = K_tile (128 x 128 e4m3) . Q_group^T (64G x 128 e4m3)
// into TMEM (M = 128 keys in lanes, N = 64G columns). The epilogue applies the
// ReLU, the w*s_q-weighted head sum, the key scale and the causal mask straight
// from TMEM, so the H^I x L x L intermediate never reaches memory; one fp32
// score per (row, key) is stored.
//
// Warp roles (384 threads):
//   warp 0      producer: TMA key tiles (2 boxes of 64 rows x 128 B, 128-B swizzle)
//               issued by lane 0, page lookups batched by the warp
//   warp 1      TMEM allocation + single-thread tcgen05.mma issue
//   warps 2-3   query quantizers: bf16 -> E4M3 rows in the canonical swizzled
//               K-major layout, w*s_q per row (double-buffered per unit)
//   warps 4-11  epilogue: two warpgroups; tiles alternate between them and
//               cycle through 512 / N TMEM accumulators (2 to 8), so the MMA
//               can run that many tiles ahead; thread = key lane, which loads
//               its key's scale from global memory itself, one tile ahead
// A stage of the ring carries key codes only and is reused as soon as the MMA has
// read it (the scales never gate a stage); the same commit tells the epilogue that
// the tile's accumulator is ready.
// Decode groups (G <= 2) run a lean form instead: two CTAs per SM, each with warps 0-2
// as above (one quantizer warp), warps 3-6 a single epilogue warpgroup, 4 key stages
// and 256 TMEM columns, so two tile pipelines share each SM.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "rows.cuh"

namespace dsa {

constexpr int kIdxHeads = 64;
constexpr int kIdxDim = 128;
constexpr int kIdxTile = 128;                      // keys per tile (MMA M)
constexpr int kIdxStages = 8;
constexpr int kIdxThreads = 384;
constexpr int kIdxStageBytes = kIdxTile * kIdxDim;  // 16 KB of e4m3
constexpr int kIdxQBufBytes = 4 * kIdxHeads * kIdxDim;  // G <= 4 rows x 64 heads x 128 B
constexpr int kIdxSmemBytes =
    1024 /*align slack*/ + kIdxStages * kIdxStageBytes + 2 * kIdxQBufBytes +
    2 * 4 * kIdxHeads * 4 /*wq*/ + 512 /*barriers etc*/ + 512 /*share + scan scratch*/ +
    2 * 4 * 256 * 4 /*filter mode: candidate keys staged for one tile*/;
constexpr int kIdxMaxAcc = 8;  // TMEM accumulators: 512 / N, at most 8
// Lean decode form (groups of at most two rows): two CTAs per SM, each with seven warps
// (producer, MMA, one quantizer, one epilogue warpgroup), four key stages and half of
// the SM's tensor memory, so that two independent tile pipelines share each SM.
constexpr int kIdxLeanThreads = 224;
constexpr int kIdxLeanStages = 4;
constexpr int kIdxLeanQBufBytes = 2 * kIdxHeads * kIdxDim;  // G <= 2 rows x 64 heads x 128 B
constexpr int kIdxLeanSmemBytes = 1024 + kIdxLeanStages * kIdxStageBytes +
                                  2 * kIdxLeanQBufBytes + 2 * 4 * kIdxHeads * 4 + 512 + 512;

struct IndexerParams {
  const __nv_bfloat16* q_idx;  // [T][64][128]
  const uint8_t* k_idx;        // [cache_rows][128] E4M3 key codes
  int64_t cache_rows;
  const float* w;              // [T][64]
  const float* k_scale;        // [cache_rows]
  const int32_t* block_table;  // [batch][max_pages] when paged
  const int32_t* seqlens;      // [batch] or nullptr
  float* scores;               // [batch * row_count][ld]
  int64_t ld;
  int32_t batch, max_ctx, q_per_seq;
  int32_t paged, page_size, max_pages, num_pages;
  int32_t row_begin, row_count;  // rows [row_begin, row_begin + row_count) of each sequence
  int32_t G;                     // query rows per MMA (N = 64 G)
  int32_t groups_per_seq;        // ceil(row_count / G)
  int32_t num_groups;            // batch * groups_per_seq
  // Strided sample: only key tiles 0, S, 2S, ... of each row (S = tile_stride >= 1);
  // sample tile u is stored at score columns [128 u, 128 u + 128).
  int32_t tile_stride;
  // Filter mode (thr != nullptr): instead of storing scores, the keys of window row
  // r whose score is >= thr[r] are appended to the row's candidate list as
  // (order-preserving key, position); cand_cnt[r] counts them (and may exceed
  // cand_cap, in which case the list holds an arbitrary cand_cap of them).
  const float* thr;
  uint32_t* cand_key;            // [batch * row_count][cand_cap]
  int32_t* cand_pos;             // [batch * row_count][cand_cap]
  uint32_t* cand_cnt;            // [batch * row_count], zeroed by the caller
  int32_t cand_cap;
  const int32_t* q_start;        // [batch + 1] ragged query rows, or nullptr (rows.cuh)
  int32_t num_q;
  uint64_t timeout_ns;
};

// One unit: key tiles [kt0, kt1) of the group (sequence b, rows i0 .. i0+nrows-1;
// the sequence has q_len query rows, the first of them global row t0).
struct IdxUnit {
  int b, i0, nrows, seqlen, q_len, kt0, kt1;
  int64_t t0;
};

// Tiles of group `grp` (0 when its sequence is invalid or has none of the group's
// rows) and its geometry.
__device__ __forceinline__ int idx_group(const IndexerParams& p, int grp, IdxUnit& U) {
  U.b = grp / p.groups_per_seq;
  const int g = grp - U.b * p.groups_per_seq;
  const SeqRows R = seq_rows(p.q_start, p.seqlens, U.b, p.q_per_seq, p.num_q, p.max_ctx);
  if (!R.ok) return 0;
  U.seqlen = R.seqlen;
  U.q_len = R.q_len;
  U.t0 = R.t0;
  U.i0 = p.row_begin + g * p.G;
  U.nrows = min(p.G, min(p.row_begin + p.row_count, R.q_len) - U.i0);
  if (U.nrows <= 0) return 0;
  const int pos_max = U.seqlen - U.q_len + U.i0 + U.nrows - 1;
  return (pos_max / kIdxTile) / p.tile_stride + 1;  // tiles 0, S, ..., up to pos_max's
}

// This CTA's share of the tile list: from (group gs, tile ts) to the exclusive
// end (group ge, tile te); every role walks the same units with IdxCursor.
struct IdxShare {
  int gs, ts, ge, te;
};
struct IdxCursor {
  int grp, kt;
};
__device__ __forceinline__ bool idx_next(const IndexerParams& p, const IdxShare& sh,
                                         IdxCursor& c, IdxUnit& U) {
  while (c.grp <= sh.ge && c.grp < p.num_groups) {
    const int nt = idx_group(p, c.grp, U);
    const int end = c.grp == sh.ge ? min(sh.te, nt) : nt;
    if (c.kt < end) {
      U.kt0 = c.kt;
      U.kt1 = end;
      ++c.grp;
      c.kt = 0;
      return true;
    }
    ++c.grp;
    c.kt = 0;
  }
  return false;
}

// Work is balanced on a cost of (tiles + G * kIdxRowCost) per group: a group's G
// query rows are quantized once per unit (64 rows of 128 elements each), which
// is worth about 8 tiles per row, so many short causal groups (early prefill
// rows) weigh what they cost. A cost position x within a group maps to the tile
// boundary max(0, x - unit cost); neighbouring shares apply the same map to
// their common boundary.
constexpr int kIdxRowCost = 8;

// Block-wide: the exact share [W c / n, W (c+1) / n) of the total cost W.
__device__ void idx_share(const IndexerParams& p, IdxShare* out, uint32_t* scratch) {
  // scratch: [32] warp sums, [32] misc
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthreads = blockDim.x, nwarps = nthreads >> 5;
  auto block_sum_scan = [&](long long v, long long& excl, long long& total) {
    long long incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    long long* ws = reinterpret_cast<long long*>(scratch);
    __syncthreads();
    if (lane == 31) ws[warp] = incl;
    __syncthreads();
    long long before = 0, all = 0;
    for (int w = 0; w < nwarps; ++w) {
      const long long x = ws[w];
      if (w < warp) before += x;
      all += x;
    }
    excl = before + incl - v;
    total = all;
  };
  const long long unit_cost = (long long)kIdxRowCost * p.G;
  auto cost_of = [&](int grp, int& nt) -> long long {
    IdxUnit U;
    nt = grp < p.num_groups ? idx_group(p, grp, U) : 0;
    return nt > 0 ? (long long)nt + unit_cost : 0;
  };
  // pass 1: total cost
  long long W = 0;
  for (int base = 0; base < p.num_groups; base += nthreads) {
    int nt;
    const long long cost = cost_of(base + tid, nt);
    long long excl, tot;
    block_sum_scan(cost, excl, tot);
    W += tot;
  }
  const long long lo = W * blockIdx.x / gridDim.x, hi = W * (blockIdx.x + 1) / gridDim.x;
  if (tid == 0) *out = IdxShare{p.num_groups, 0, -1, 0};  // empty unless found below
  __syncthreads();
  if (lo >= hi) return;
  // pass 2: locate the groups holding cost positions lo and hi - 1
  long long run = 0;
  for (int base = 0; base < p.num_groups; base += nthreads) {
    const int grp = base + tid;
    int nt;
    const long long cost = cost_of(grp, nt);
    long long excl, tot;
    block_sum_scan(cost, excl, tot);
    const long long a = run + excl, e = a + cost;  // cost positions [a, e) belong to grp
    if (cost > 0 && a <= lo && lo < e) {
      out->gs = grp;
      out->ts = (int)max(0ll, lo - a - unit_cost);
    }
    if (cost > 0 && a < hi && hi <= e) {
      out->ge = grp;
      out->te = (int)max(0ll, hi - a - unit_cost);
    }
    run += tot;
  }
  __syncthreads();
}

// kFilter: the fused selection's filter mode (thr, cand_* set; no score rows); the
// plain instantiation carries none of its code.
// kLean (groups of at most 2 query rows, i.e. decode): two CTAs per SM with 7 warps
// each (warps 3-6 one epilogue warpgroup that takes every tile), 4 key stages and 256
// TMEM columns; 2 x 224 threads leave 144 registers per thread, so the epilogue reads
// tensor memory in 16-column chunks.
template <bool kFilter, bool kLean = false>
__global__ void __launch_bounds__(kLean ? kIdxLeanThreads : kIdxThreads, kLean ? 2 : 1)
    indexer_kernel(const __grid_constant__ IndexerParams p,
                   const __grid_constant__ CUtensorMap tm_keys) {
  static_assert(!(kLean && kFilter), "the lean form is for plain scores");
  constexpr int kS = kLean ? kIdxLeanStages : kIdxStages;        // key stages
  constexpr int kQB = kLean ? kIdxLeanQBufBytes : kIdxQBufBytes;  // one query buffer
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* qbuf = stages + kS * kIdxStageBytes;
  float* wq = reinterpret_cast<float*>(qbuf + 2 * kQB);  // [2][256]
  uint64_t* bars = reinterpret_cast<uint64_t*>(wq + 2 * 4 * kIdxHeads);
  uint64_t* kfull = bars;
  // kempty[s]: the MMAs of the tile in stage s are done, so its key stage is free and
  // its accumulator holds the scores (one commit per tile serves the producer and the
  // epilogue; the epilogue of a tile always observes that phase before the next tile
  // in the same stage can finish, because that tile needs the accumulator this
  // epilogue or a later one of the same warpgroup frees)
  uint64_t* kempty = bars + kS;
  uint64_t* tempty = bars + 2 * kS + kIdxMaxAcc;
  uint64_t* qfull = tempty + kIdxMaxAcc;
  uint64_t* qempty = qfull + 2;
  uint64_t* mdone = qempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mdone + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  IdxShare* share = reinterpret_cast<IdxShare*>(tmem_holder + 4);
  uint32_t* scan_scratch = reinterpret_cast<uint32_t*>(share + 1) + 4;  // 8-B aligned, 32 x i64
  // filter mode: [2 tiles][4 rows][256 epilogue threads] keys awaiting their slots
  uint32_t* cstage = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(bars) + 1024);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = kIdxHeads * p.G;
  // As many accumulators as tensor memory holds (an even number, so a given
  // accumulator always belongs to the same epilogue warpgroup): the MMA runs
  // up to nacc tiles ahead of the epilogue.
  const uint32_t tmem_cols = kLean ? 256 : 512;
  const int nacc = min(kIdxMaxAcc, (int)tmem_cols / N) & ~1;

  if (tid == 0) {
    for (int s = 0; s < kS; ++s) {
      // expect_tx arrival (+ the TMA bytes), and one arrival per copy thread
      mbar_init(smem_u32(&kfull[s]), 1);  // the producer's expect_tx arrival (+ TMA bytes)
      mbar_init(smem_u32(&kempty[s]), 1);  // the MMA's commit (stage free, scores ready)
    }
    for (int i = 0; i < kIdxMaxAcc; ++i) mbar_init(smem_u32(&tempty[i]), 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&qfull[i]), kLean ? 32 : 64);  // the quantizer warps' lanes
      mbar_init(smem_u32(&qempty[i]), 1 + (kLean ? 128 : 256));  // MMA commit + epilogue
    }
    mbar_init(smem_u32(mdone), 1);
    *abort_flag = 0;
    fence_mbarrier_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  idx_share(p, share, scan_scratch);  // ends with a barrier
  const IdxShare sh = *share;
  const uint32_t tmem_base = *tmem_holder;
  const uint64_t TO = p.timeout_ns;
  int drain_dummy = 0;
  volatile int* no_abort = &drain_dummy;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) prefetch_tmap(&tm_keys);
    uint32_t it = 0;
    IdxCursor cur{sh.gs, sh.ts};
    IdxUnit U;
    while (!*abort_flag && idx_next(p, sh, cur, U)) {
      const int pos_max = U.seqlen - U.q_len + U.i0 + U.nrows - 1;
      bool ok = true;
      // Paged caches: lane l holds the page of half (l & 1) of tile kb + l / 2
      // for a batch of 16 tiles starting at kb, and the next batch is already
      // in flight, so no tile waits on a block-table load.
      auto fetch_pages = [&](int kb) -> int {
        const int kt = kb + (lane >> 1), s0 = kt * p.tile_stride * kIdxTile + (lane & 1) * 64;
        if (!p.paged || kt >= U.kt1 || s0 > pos_max) return -1;
        return __ldg(p.block_table + (int64_t)U.b * p.max_pages + s0 / p.page_size);
      };
      int kb = U.kt0;
      int pg_cur = fetch_pages(kb), pg_nxt = fetch_pages(kb + 16);
      for (int kt = U.kt0; kt < U.kt1; ++kt, ++it) {
        if (kt - kb == 16) {
          kb = kt;
          pg_cur = pg_nxt;
          pg_nxt = fetch_pages(kb + 16);
        }
        const int st = it % kS;
        if (!warp_wait(smem_u32(&kempty[st]), ((it / kS) & 1) ^ 1, TO, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t bar = smem_u32(&kfull[st]);
        // cache rows of the tile's two 64-key halves (a half never straddles a page)
        int64_t base[2] = {0, 0};  // half tiles past pos_max or behind a bad page load row 0
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int s0 = kt * p.tile_stride * kIdxTile + h * 64;
          const int page = __shfl_sync(0xffffffffu, pg_cur, 2 * (kt - kb) + h);
          if (s0 <= pos_max) {
            if (!p.paged) {
              base[h] = (int64_t)U.b * p.max_ctx + s0;
            } else if (page >= 0 && page < p.num_pages) {
              base[h] = (int64_t)page * p.page_size + s0 % p.page_size;
            } else if (lane == 0) {
              report_error(kErrBounds);
            }
          }
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(bar, kIdxStageBytes);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tma_load_2d(smem_u32(stages + st * kIdxStageBytes + h * 8192), &tm_keys, bar, 0,
                        (int)base[h]);
        }
      }
      if (!ok) break;
    }
    // Drain: the last stages' copies must land before the CTA may exit.
    if (lane == 0)
      for (uint32_t j = it > kS ? it - kS : 0; j < it; ++j)
        mbar_wait(smem_u32(&kfull[j % kS]), (j / kS) & 1, TO, no_abort);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = instr_desc(0 /*e4m3*/, 0, 0, 128, N);
      uint32_t it = 0, un = 0;
      IdxCursor cur{sh.gs, sh.ts};
      IdxUnit U;
      while (!*abort_flag && idx_next(p, sh, cur, U)) {
        const int qb = un & 1;
        if (!mbar_wait(smem_u32(&qfull[qb]), (un >> 1) & 1, TO, abort_flag)) break;
        const uint32_t qaddr = smem_u32(qbuf + qb * kQB);
        bool ok = true;
        for (int kt = U.kt0; kt < U.kt1; ++kt, ++it) {
          const int st = it % kS, ab = it % nacc;
          if (!mbar_wait(smem_u32(&kfull[st]), (it / kS) & 1, TO, abort_flag) ||
              !mbar_wait(smem_u32(&tempty[ab]), ((it / nacc) & 1) ^ 1, TO, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kaddr = smem_u32(stages + st * kIdxStageBytes);
          const uint32_t dcol = tmem_base + ab * N;
#pragma unroll
          for (int kk = 0; kk < kIdxDim / 32; ++kk) {
            const uint64_t adesc = smem_desc_sw128(kaddr + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(qaddr + kk * 32, 16, 1024);
            mma_fp8_ss(dcol, adesc, bdesc, idesc, kk > 0);
          }
          mma_commit(smem_u32(&kempty[st]));
        }
        if (!ok) break;
        mma_commit(smem_u32(&qempty[qb]));
        ++un;
      }
      // Every MMA issued above must finish before TMEM may be released.
      mma_commit(smem_u32(mdone));
      mbar_wait(smem_u32(mdone), 0, TO, no_abort);
    }
    __syncwarp();
  } else if (kLean ? warp == 2 : warp < 4) {
    // ------------------------------------------------------------ query quantizers
    const int qw = warp - 2;  // 0..1 (the lean form has warp 2 only)
    constexpr int kQW = kLean ? 1 : 2;  // quantizer warps
    uint32_t un = 0;
    IdxCursor cur{sh.gs, sh.ts};
    IdxUnit U;
    while (!*abort_flag && idx_next(p, sh, cur, U)) {
      const int qb = un & 1;
      if (!warp_wait(smem_u32(&qempty[qb]), ((un >> 1) & 1) ^ 1, TO, abort_flag)) break;
      uint8_t* qdst = qbuf + qb * kQB;
      float* wdst = wq + qb * 4 * kIdxHeads;
      // A half-warp converts one 128-element row (8 elements = 16 B per lane);
      // kQRows rows per half-warp are loaded before any is used, so their
      // global load latencies overlap (the loads compete with every CTA's key
      // stream, so each round trip is long). Rows r = base + 4 i of the batch.
      constexpr int kQRows = 16;
      const int half = lane >> 4, hl = lane & 15;
      for (int base = qw * 2 + half; base < N; base += 2 * kQW * kQRows) {
        uint4 raw[kQRows];
        float wj[kQRows];
#pragma unroll
        for (int i = 0; i < kQRows; ++i) {
          const int r = base + 2 * kQW * i;
          const int gi = r / kIdxHeads, j = r % kIdxHeads;
          raw[i] = make_uint4(0u, 0u, 0u, 0u);
          wj[i] = 0.f;
          if (gi < U.nrows) {
            const int64_t t = U.t0 + U.i0 + gi;
            raw[i] = __ldg(reinterpret_cast<const uint4*>(p.q_idx + (t * kIdxHeads + j) * kIdxDim) +
                           hl);
            wj[i] = __ldg(p.w + t * kIdxHeads + j);
          }
        }
#pragma unroll
        for (int i = 0; i < kQRows; ++i) {
          const int r = base + 2 * kQW * i;  // < N: N is a multiple of 64
          const uint32_t wv[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
          float x[8];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            x[2 * c] = __uint_as_float(wv[c] << 16);
            x[2 * c + 1] = __uint_as_float(wv[c] & 0xFFFF0000u);
          }
          float amax = 0.f;
#pragma unroll
          for (int c = 0; c < 8; ++c) amax = fmaxf(amax, fabsf(x[c]));
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
          const float sq = __fdiv_rn(fmaxf(amax, 0x1p-120f), 448.0f);
          uint32_t code[4];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            code[c] = cvt_e4m3x2(__fdiv_rn(x[2 * c], sq), __fdiv_rn(x[2 * c + 1], sq));
          *reinterpret_cast<uint2*>(qdst + sw128_offset(r, hl >> 1) + (hl & 1) * 8) =
              make_uint2(code[0] | (code[1] << 16), code[2] | (code[3] << 16));
          if (hl == 0) wdst[r] = wj[i] * sq;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&qfull[qb]));
      ++un;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int wg = kLean ? 0 : (warp - 4) >> 2;  // warpgroup: takes every other tile
    const int quad = warp & 3;         // TMEM lane quadrant of this warp
    const int e = quad * 32 + lane;    // key within the tile == TMEM lane
    const int et = tid - 4 * 32;       // 0..255 among the epilogue threads (filter mode)
    constexpr int kNext = kLean ? 1 : 2;  // this warpgroup's next tile
    int cpar = 0;                      // filter mode: staging buffer of the next tile
    uint32_t it = 0, un = 0;
    if (blockIdx.x == 0 && wg == 0) {  // sequences whose rows or length are out of range
      for (int b = e; b < p.batch; b += 128)
        if (!seq_rows(p.q_start, p.seqlens, b, p.q_per_seq, p.num_q, p.max_ctx).ok)
          report_error(kErrBounds);
    }
    IdxCursor cur{sh.gs, sh.ts};
    IdxUnit U;
    while (!*abort_flag && idx_next(p, sh, cur, U)) {
      const int qb = un & 1;
      if (!warp_wait(smem_u32(&qfull[qb]), (un >> 1) & 1, TO, abort_flag)) break;
      const float* wrow = wq + qb * 4 * kIdxHeads;
      const int pos0 = U.seqlen - U.q_len + U.i0;  // position of the group's first row
      const int pos_max = pos0 + U.nrows - 1;
      float thr_row[4] = {0.f, 0.f, 0.f, 0.f};  // filter mode: the rows' thresholds
      if (kFilter)
        for (int gi = 0; gi < U.nrows; ++gi)
          thr_row[gi] = __ldg(p.thr + (int64_t)U.b * p.row_count + (U.i0 - p.row_begin) + gi);
      // this thread's key scale of tile kt (0 past the last visible key or behind
      // an invalid page entry, whose scores are masked or reported anyway)
      auto scale_of = [&](int kt) -> float {  // kt: the unit's tile index (strided)
        const int s = kt * p.tile_stride * kIdxTile + e;
        if (s > pos_max) return 0.f;
        int64_t row = (int64_t)U.b * p.max_ctx + s;
        if (p.paged) {
          const int pg = __ldg(p.block_table + (int64_t)U.b * p.max_pages + s / p.page_size);
          if (pg < 0 || pg >= p.num_pages) return 0.f;
          row = (int64_t)pg * p.page_size + s % p.page_size;
        }
        return __ldg(p.k_scale + row);
      };
      int pf_kt = -1;  // the tile whose scale is already in flight (this warpgroup's next)
      float pf_ks = 0.f;
      // Filter mode: a tile's candidates reserve their slots (one atomic per warp and
      // row) after its rows are reduced, and are written one tile later, so the
      // atomic's round trip overlaps the next tile instead of stalling the warp.
      const int64_t orow0 = (int64_t)U.b * p.row_count + (U.i0 - p.row_begin);
      uint32_t pend_bal[4] = {0u, 0u, 0u, 0u}, pend_base[4] = {0u, 0u, 0u, 0u};
      uint32_t pend_bits = 0;
      int pend_s = 0, pend_par = 0;
      auto flush = [&]() {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint32_t bal = pend_bal[g];
          if (bal) {  // warp-uniform
            const uint32_t base = __shfl_sync(0xffffffffu, pend_base[g], __ffs(bal) - 1);
            const uint32_t slot = base + __popc(bal & ((1u << lane) - 1u));
            if (((pend_bits >> g) & 1u) && slot < (uint32_t)p.cand_cap) {
              p.cand_key[(orow0 + g) * p.cand_cap + slot] = cstage[((pend_par * 4 + g) << 8) + et];
              p.cand_pos[(orow0 + g) * p.cand_cap + slot] = pend_s;
            }
          }
          pend_bal[g] = 0u;
        }
      };
      bool ok = true;
      for (int kt = U.kt0; kt < U.kt1; ++kt, ++it) {
        if (!kLean && (int)(it & 1) != wg) continue;  // the other warpgroup's tile
        const int s = kt * p.tile_stride * kIdxTile + e;  // this thread's key
        const float ks = pf_kt == kt ? pf_ks : scale_of(kt);
        if (kt + kNext < U.kt1) {
          pf_ks = scale_of(kt + kNext);
          pf_kt = kt + kNext;
        }
        const int ab = (int)(it % (uint32_t)nacc);  // accumulator of this tile
        if (!warp_wait(smem_u32(&kempty[it % kS]), (it / kS) & 1, TO, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tcol = tmem_base + ((uint32_t)(quad * 32) << 16) + ab * N;
        uint32_t take_bits = 0;  // filter mode: rows that keep this thread's key
        // row gi's score from its weighted head sum: causal mask, key scale, then the
        // score row (or, in filter mode, the candidate note)
        auto finish_row = [&](int gi, float acc) {
          const float out = (s <= pos0 + gi) ? ks * acc : -INFINITY;
          const int64_t orow = (int64_t)U.b * p.row_count + (U.i0 - p.row_begin) + gi;
          if (!kFilter) {
            p.scores[orow * p.ld + kt * kIdxTile + e] = out;
          } else {  // filter mode: note the key; its slot is reserved after the rows
            const bool take = s <= pos0 + gi && out >= thr_row[gi];
            take_bits |= (take ? 1u : 0u) << gi;
            cstage[((cpar * 4 + gi) << 8) + et] = score_key(out);
          }
        };
        if constexpr (kLean) {
          // 16-column chunks (the two-CTA form's register budget): row gi's 64 head
          // columns as four chunks, the next one's load in flight while one is reduced
          uint32_t ca[16], cb[16];
          tmem_ld16u(tcol, ca);
          tmem_wait_ld_fence16(ca);
          for (int gi = 0; gi < U.nrows; ++gi) {
            const float4* w4 = reinterpret_cast<const float4*>(wrow + gi * kIdxHeads);
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            auto reduce16 = [&](const uint32_t (&v)[16], const float4* wq4) {
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const float4 wv = wq4[q4];
                a0 = fmaf(wv.x, fmaxf(__uint_as_float(v[4 * q4 + 0]), 0.f), a0);
                a1 = fmaf(wv.y, fmaxf(__uint_as_float(v[4 * q4 + 1]), 0.f), a1);
                a2 = fmaf(wv.z, fmaxf(__uint_as_float(v[4 * q4 + 2]), 0.f), a2);
                a3 = fmaf(wv.w, fmaxf(__uint_as_float(v[4 * q4 + 3]), 0.f), a3);
              }
            };
            const uint32_t rc = tcol + gi * kIdxHeads;
            tmem_ld16u(rc + 16, cb);
            reduce16(ca, w4);
            tmem_wait_ld_fence16(cb);
            tmem_ld16u(rc + 32, ca);
            reduce16(cb, w4 + 4);
            tmem_wait_ld_fence16(ca);
            tmem_ld16u(rc + 48, cb);
            reduce16(ca, w4 + 8);
            tmem_wait_ld_fence16(cb);
            if (gi + 1 < U.nrows) tmem_ld16u(tcol + (gi + 1) * kIdxHeads, ca);
            reduce16(cb, w4 + 12);
            if (gi + 1 < U.nrows) tmem_wait_ld_fence16(ca);
            finish_row(gi, (a0 + a1) + (a2 + a3));
          }
        } else {
          // Row gi's 64 head columns come as two 32-column chunks (A: heads 0-31, B:
          // heads 32-63). The next chunk's load is always in flight while the current
          // one is reduced, so the tensor-memory load latency hides behind the ReLU /
          // weighted head sum.
          uint32_t ca[32], cb[32];
          tmem_ld32u(tcol, ca);
          tmem_wait_ld_fence(ca);
          for (int gi = 0; gi < U.nrows; ++gi) {
            const float4* w4 = reinterpret_cast<const float4*>(wrow + gi * kIdxHeads);
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            auto reduce32 = [&](const uint32_t (&v)[32], const float4* wq4) {
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4) {
                const float4 wv = wq4[q4];
                a0 = fmaf(wv.x, fmaxf(__uint_as_float(v[4 * q4 + 0]), 0.f), a0);
                a1 = fmaf(wv.y, fmaxf(__uint_as_float(v[4 * q4 + 1]), 0.f), a1);
                a2 = fmaf(wv.z, fmaxf(__uint_as_float(v[4 * q4 + 2]), 0.f), a2);
                a3 = fmaf(wv.w, fmaxf(__uint_as_float(v[4 * q4 + 3]), 0.f), a3);
              }
            };
            tmem_ld32u(tcol + gi * kIdxHeads + 32, cb);
            reduce32(ca, w4);
            tmem_wait_ld_fence(cb);
            if (gi + 1 < U.nrows) tmem_ld32u(tcol + (gi + 1) * kIdxHeads, ca);
            reduce32(cb, w4 + 8);
            if (gi + 1 < U.nrows) tmem_wait_ld_fence(ca);
            finish_row(gi, (a0 + a1) + (a2 + a3));
          }
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&tempty[ab]));
        if (kFilter) {
          flush();  // the previous tile's candidates: their slots have arrived by now
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint32_t bal =
                __ballot_sync(0xffffffffu, g < U.nrows && ((take_bits >> g) & 1u));
            pend_bal[g] = bal;
            pend_base[g] = 0u;
            if (bal && lane == __ffs(bal) - 1)
              pend_base[g] = atomicAdd(p.cand_cnt + orow0 + g, __popc(bal));
          }
          pend_bits = take_bits;
          pend_s = s;
          pend_par = cpar;
          cpar ^= 1;
        }
      }
      if (!ok) break;
      if (kFilter) flush();  // the unit's last tile
      mbar_arrive(smem_u32(&qempty[qb]));
      ++un;
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

}  // namespace dsa
