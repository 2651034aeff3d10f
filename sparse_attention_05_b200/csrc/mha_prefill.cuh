// mha_prefill.cuh -- MLA in MHA mode: the masked-MHA emulation of DSA for short prefill.
//
// DeepSeek-V3.2-Exp technical report (zh translation), Appendix A and Fig. 4: MLA
// has an MHA mode (training and prefill) and an MQA mode (decode), related by
// absorbing the up-projections. §3 "Inference cost": for short-sequence prefill
// a masked MHA mode emulates DSA, which is cheaper in short contexts.
//
// MHA mode per head h (128 heads): key k_{h,s} = [W^UK_h c_s[0:512] ; c_s[512:576]]
// (128 nope dims from the latent, the 64 rope dims shared by every head), value
// v_{h,s} = W^UV_h c_s[0:512] (128 dims), query q_{t,h} = [q^C (128) ; q^R (64)].
// Row t of head h attends over the keys its selection S_t admits (plain causal
// when every visible key is selected, i.e. pos(t) + 1 <= k). A (t, s) pair costs
// 2 * 128 * (192 + 128) = 81920 FLOP here against 278528 in MQA mode, and the
// key/value tiles are dense, so the work maps onto full tensor-core tiles.
//
// Three kernels:
//   mla_up_proj_kernel   [keys x 512] . [512 x 256] per (128-key tile, head):
//                        tcgen05 BF16 GEMM, N = 256 (the head's 128 key and
//                        128 value outputs), K-chunks of 64 latent dims through
//                        a 4-stage TMA ring, two TMEM accumulators so the
//                        epilogue of one tile overlaps the MMAs of the next;
//                        keys past the sequence end are written as zeros.
//   selection_mask_kernel  the selected index list of a row -> a bitmask over
//                        its keys (only rows with more than k visible keys).
//   masked_mha_kernel    flash attention over the decompressed keys/values: one
//                        CTA per (sequence, head, 128 query rows); per 128-key
//                        tile S = Q K^T (M = 128 rows, N = 128 keys, K = 192)
//                        into one of two TMEM score buffers, an online softmax
//                        in base 2 with a lazy rescale of O (only when the
//                        running max grows by more than 8), P written back as
//                        bf16 into the score buffer, O += P V with P from TMEM.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "rows.cuh"

namespace dsa {

constexpr int kMhaHeads = 128;
constexpr int kMhaDc = 512;      // latent dims that pass through the up-projections
constexpr int kMhaDr = 64;       // rope dims, shared by all heads
constexpr int kMhaDn = 128;      // nope query/key dims per head
constexpr int kMhaDqk = kMhaDn + kMhaDr;
constexpr int kMhaDv = 128;      // value dims per head
constexpr int kMhaLat = 576;     // latent cache row
constexpr int kMhaTile = 128;    // keys per tile, query rows per CTA

// ======================================================================================
// Up-projection
// ======================================================================================
constexpr int kUpStages = 4;
constexpr int kUpChunkA = kMhaTile * 128;          // 128 keys x 64 latent dims (16 KB)
constexpr int kUpChunkB = 2 * kMhaDn * 128;        // 256 outputs x 64 latent dims (32 KB)
constexpr int kUpStageBytes = kUpChunkA + kUpChunkB;
constexpr int kUpChunks = kMhaDc / 64;             // 8 K-chunks
constexpr int kUpThreads = 192;                    // TMA, MMA + TMEM, 4 epilogue warps
constexpr int kUpSmemBytes = 1024 + kUpStages * kUpStageBytes + 256;

struct UpProjParams {
  const int32_t* block_table;  // [batch][max_pages] when paged
  const int32_t* seqlens;      // [batch] or nullptr
  const __nv_bfloat16* kv;     // latent cache rows [cache_rows][576]
  __nv_bfloat16* k_nope;       // [batch][128][ctx_pad][128]
  __nv_bfloat16* k_rope;       // [batch][ctx_pad][64]
  __nv_bfloat16* v;            // [batch][128][ctx_pad][128]
  int64_t ctx_pad;             // key_tiles * 128
  int32_t batch, max_ctx, q_per_seq, paged, page_size, max_pages, num_pages;
  int32_t key_tiles;
  uint64_t timeout_ns;
};

// Latent cache row of token s of sequence b, or -1 when its page entry is invalid.
__device__ __forceinline__ int64_t mha_latent_row(const int32_t* block_table, int paged,
                                                  int page_size, int max_pages, int num_pages,
                                                  int max_ctx, int b, int s) {
  if (!paged) return (int64_t)b * max_ctx + s;
  const int pg = __ldg(block_table + (int64_t)b * max_pages + s / page_size);
  if (pg < 0 || pg >= num_pages) return -1;
  return (int64_t)pg * page_size + s % page_size;
}

__device__ __forceinline__ int mha_seqlen(const int32_t* seqlens, int b, int max_ctx) {
  return seqlens ? __ldg(seqlens + b) : max_ctx;
}

// Work item i -> (sequence, key tile, head), heads fastest so that the CTAs running
// at the same time share one latent tile; false when the tile lies past the end.
__device__ __forceinline__ bool up_item(const UpProjParams& p, int64_t i, int& b, int& kt,
                                        int& h, int& seqlen) {
  h = (int)(i % kMhaHeads);
  const int64_t r = i / kMhaHeads;
  kt = (int)(r % p.key_tiles);
  b = (int)(r / p.key_tiles);
  seqlen = mha_seqlen(p.seqlens, b, p.max_ctx);
  return seqlen >= 1 && seqlen <= p.max_ctx && kt * kMhaTile < seqlen;
}

__global__ void __launch_bounds__(kUpThreads, 1)
    mla_up_proj_kernel(const UpProjParams p, const __grid_constant__ CUtensorMap tm_lat,
                       const __grid_constant__ CUtensorMap tm_uk,
                       const __grid_constant__ CUtensorMap tm_uv) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sStage = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kUpStages * kUpStageBytes);
  uint64_t* empty = full + kUpStages;
  uint64_t* tfull = empty + kUpStages;  // [2] accumulator ready
  uint64_t* tempty = tfull + 2;         // [2] accumulator drained by the epilogue
  uint64_t* mdone = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mdone + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < kUpStages; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), 128);
    }
    mbar_init(smem_u32(mdone), 1);
    *abort_flag = 0;
    fence_mbarrier_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint64_t TO = p.timeout_ns;
  int drain_dummy = 0;
  volatile int* no_abort = &drain_dummy;
  const int64_t n_items = (int64_t)p.batch * p.key_tiles * kMhaHeads;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int issued = 0;
    if (lane == 0) {
      prefetch_tmap(&tm_lat);
      prefetch_tmap(&tm_uk);
      prefetch_tmap(&tm_uv);
      bool ok = true;
      for (int64_t i = blockIdx.x; ok && i < n_items; i += gridDim.x) {
        int b, kt, h, seqlen;
        if (!up_item(p, i, b, kt, h, seqlen)) continue;
        // the two 64-key halves of the tile (a page holds whole halves); rows past
        // the sequence end or behind an invalid page entry load as zeros (row -64)
        int y[2];
        for (int half = 0; half < 2; ++half) {
          const int s0 = kt * kMhaTile + 64 * half;
          int64_t row = -64;
          if (s0 < seqlen) {
            row = mha_latent_row(p.block_table, p.paged, p.page_size, p.max_pages, p.num_pages,
                                 p.max_ctx, b, s0);
            if (row < 0) {
              report_error(kErrBounds);
              row = -64;
            }
          }
          y[half] = (int)row;
        }
        for (int c = 0; c < kUpChunks; ++c, ++issued) {
          const int st = issued % kUpStages;
          ok = mbar_wait(smem_u32(&empty[st]), ((issued / kUpStages) & 1) ^ 1, TO, abort_flag);
          if (!ok) break;
          const uint32_t bar = smem_u32(&full[st]);
          const uint32_t a = smem_u32(sStage + st * kUpStageBytes);
          mbar_arrive_expect_tx(bar, kUpStageBytes);
          tma_load_2d(a, &tm_lat, bar, 64 * c, y[0]);
          tma_load_2d(a + kUpChunkA / 2, &tm_lat, bar, 64 * c, y[1]);
          tma_load_2d(a + kUpChunkA, &tm_uk, bar, 64 * c, h * kMhaDn);
          tma_load_2d(a + kUpChunkA + kUpChunkB / 2, &tm_uv, bar, 64 * c, h * kMhaDv);
        }
      }
      // on an early exit, let the copies still in flight land before the CTA can leave
      for (int j = issued > kUpStages ? issued - kUpStages : 0; j < issued; ++j)
        mbar_wait(smem_u32(&full[j % kUpStages]), (j / kUpStages) & 1, TO, no_abort);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = instr_desc(1 /*bf16*/, 0, 0, 128, 2 * kMhaDn);
      int used = 0, n = 0;
      bool ok = true;
      for (int64_t i = blockIdx.x; ok && i < n_items; i += gridDim.x) {
        int b, kt, h, seqlen;
        if (!up_item(p, i, b, kt, h, seqlen)) continue;
        const int acc = n & 1;
        ok = mbar_wait(smem_u32(&tempty[acc]), ((n >> 1) & 1) ^ 1, TO, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * 2 * kMhaDn);
        for (int c = 0; c < kUpChunks && ok; ++c, ++used) {
          const int st = used % kUpStages;
          ok = mbar_wait(smem_u32(&full[st]), (used / kUpStages) & 1, TO, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a = smem_u32(sStage + st * kUpStageBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(d, smem_desc_sw128(a + kk * 32, 16, 1024),
                        smem_desc_sw128(a + kUpChunkA + kk * 32, 16, 1024), idesc,
                        (c > 0 || kk > 0) ? 1u : 0u);
          mma_commit(smem_u32(&empty[st]));
        }
        if (ok) mma_commit(smem_u32(&tfull[acc]));
        ++n;
      }
      mma_commit(smem_u32(mdone));
      mbar_wait(smem_u32(mdone), 0, TO, no_abort);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // thread = key lane of the accumulator (TMEM lane quadrant = warp % 4)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    int n = 0;
    bool ok = true;
    for (int64_t i = blockIdx.x; ok && i < n_items; i += gridDim.x) {
      int b, kt, h, seqlen;
      if (!up_item(p, i, b, kt, h, seqlen)) continue;
      const int acc = n & 1;
      ok = warp_wait(smem_u32(&tfull[acc]), (n >> 1) & 1, TO, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const int s = kt * kMhaTile + r;
      const bool valid = s < seqlen;
      const int64_t kv_row = ((int64_t)b * kMhaHeads + h) * p.ctx_pad + s;
      uint4* dk = reinterpret_cast<uint4*>(p.k_nope + kv_row * kMhaDn);
      uint4* dv = reinterpret_cast<uint4*>(p.v + kv_row * kMhaDv);
      const uint32_t tacc = tmem_base + (uint32_t)(acc * 2 * kMhaDn) + lane_off;
#pragma unroll 1
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t x[32];
        tmem_ld32u(tacc + cc * 32, x);
        tmem_wait_ld_fence(x);
        uint4* dst = (cc < 4 ? dk : dv) + (cc & 3) * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 o = make_uint4(0, 0, 0, 0);
          if (valid)
            o = make_uint4(pack_bf16x2(__uint_as_float(x[8 * q]), __uint_as_float(x[8 * q + 1])),
                           pack_bf16x2(__uint_as_float(x[8 * q + 2]), __uint_as_float(x[8 * q + 3])),
                           pack_bf16x2(__uint_as_float(x[8 * q + 4]), __uint_as_float(x[8 * q + 5])),
                           pack_bf16x2(__uint_as_float(x[8 * q + 6]), __uint_as_float(x[8 * q + 7])));
          dst[q] = o;
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&tempty[acc]));
      if (h == 0) {
        // the shared rope dims of the key, once per token
        uint4* dr = reinterpret_cast<uint4*>(p.k_rope + ((int64_t)b * p.ctx_pad + s) * kMhaDr);
        int64_t row = -1;
        if (valid)
          row = mha_latent_row(p.block_table, p.paged, p.page_size, p.max_pages, p.num_pages,
                               p.max_ctx, b, s);
        if (row >= 0) {
          const uint4* src = reinterpret_cast<const uint4*>(p.kv + row * kMhaLat + kMhaDc);
#pragma unroll
          for (int q = 0; q < 8; ++q) dr[q] = __ldg(src + q);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) dr[q] = make_uint4(0, 0, 0, 0);
        }
      }
      ++n;
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ======================================================================================
// Selection mask
// ======================================================================================
constexpr int kMaskThreads = 256;

struct MaskParams {
  const int32_t* idx;      // [T][k] selected positions (global query rows)
  const int32_t* seqlens;  // [batch] or nullptr
  uint32_t* mask;          // [T][mask_ld] bits, row t = the global query row
  int64_t mask_ld;         // words per mask row (>= 4 * key tiles)
  int32_t k, batch, max_ctx, q_per_seq, row_begin, row_count;
  const int32_t* q_start;  // [batch + 1] ragged query rows, or nullptr (rows.cuh)
  int32_t num_q;
};

// One CTA per window row. Rows with at most k visible keys select all of them and
// are left untouched (the attention kernel treats them as causal). Entries outside
// [0, pos] are ignored and a position listed twice counts once.
__global__ void __launch_bounds__(kMaskThreads)
    selection_mask_kernel(const MaskParams p) {
  extern __shared__ uint32_t sbits[];
  const int b = (int)(blockIdx.x / p.row_count);
  const int qi = p.row_begin + (int)(blockIdx.x - (int64_t)b * p.row_count);
  const SeqRows R = seq_rows(p.q_start, p.seqlens, b, p.q_per_seq, p.num_q, p.max_ctx);
  if (!R.ok || qi >= R.q_len) return;  // the attention reports a bad sequence
  const int64_t t = R.t0 + qi;
  const int pos = R.seqlen - R.q_len + qi;
  if (pos + 1 <= p.k) return;
  const int words = ((pos + kMhaTile) / kMhaTile) * 4;  // whole 128-key tiles up to pos
  for (int w = threadIdx.x; w < words; w += kMaskThreads) sbits[w] = 0u;
  __syncthreads();
  const int32_t* sel = p.idx + t * p.k;
  for (int i = threadIdx.x; i < p.k; i += kMaskThreads) {
    const int s = __ldg(sel + i);
    if (s >= 0 && s <= pos) atomicOr(&sbits[s >> 5], 1u << (s & 31));
  }
  __syncthreads();
  uint4* dst = reinterpret_cast<uint4*>(p.mask + t * p.mask_ld);
  for (int w = threadIdx.x; w < words / 4; w += kMaskThreads)
    dst[w] = make_uint4(sbits[4 * w], sbits[4 * w + 1], sbits[4 * w + 2], sbits[4 * w + 3]);
}

// ======================================================================================
// Masked MHA (flash attention over decompressed keys / values)
// ======================================================================================
constexpr int kFaQChunk = kMhaTile * 128;            // 128 rows x 64 dims (16 KB)
constexpr int kFaQBytes = 3 * kFaQChunk;             // Q: nope 0-63, nope 64-127, rope
constexpr int kFaKBytes = 3 * kFaQChunk;             // a key tile, same three chunks
constexpr int kFaVBytes = 2 * kFaQChunk;             // a value tile: dims 0-63, 64-127
constexpr int kFaThreads = 224;  // K producer, MMA + TMEM, 4 softmax warps, V producer
constexpr int kFaSmemBytes = 1024 + kFaQBytes + 2 * kFaKBytes + 2 * kFaVBytes + 256;
constexpr uint32_t kFaTmemO = 256;                   // S0 at 0, S1 at 128, O at 256

struct MhaParams {
  const int32_t* seqlens;  // [batch] or nullptr
  const uint32_t* mask;    // [T][mask_ld] selection bits or nullptr (all rows causal)
  __nv_bfloat16* out;      // [T][128][128]
  float* lse;              // [T][128]
  int64_t ctx_pad, mask_ld;
  int32_t batch, max_ctx, q_per_seq, row_begin, row_count, row_blocks, k;
  float scale_log2;        // softmax scale * log2(e)
  uint64_t timeout_ns;
  const int32_t* q_start;  // [batch + 1] ragged query rows, or nullptr (rows.cuh)
  int32_t num_q;
};

__global__ void __launch_bounds__(kFaThreads, 1)
    masked_mha_kernel(const MhaParams p, const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_kn,
                      const __grid_constant__ CUtensorMap tm_kr,
                      const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kFaQBytes;           // [2]
  uint8_t* sV = sK + 2 * kFaKBytes;       // [2]
  uint64_t* qfull = reinterpret_cast<uint64_t*>(sV + 2 * kFaVBytes);
  uint64_t* kfull = qfull + 1;            // [2]
  uint64_t* kempty = kfull + 2;           // [2] S of the tile issued (keys read)
  uint64_t* vfull = kempty + 2;           // [2]
  uint64_t* vempty = vfull + 2;           // [2] P.V of the tile done (values read)
  uint64_t* sfull = vempty + 2;           // [2] scores in TMEM
  uint64_t* pfull = sfull + 2;            // [2] P in TMEM, O rescaled (128 arrivals)
  uint64_t* odone = pfull + 2;            // one phase per P.V
  uint64_t* mdone = odone + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mdone + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Head-major order: the CTAs resident together are the row blocks of one or two
  // (sequence, head) pairs, which read the same key/value tiles, so each tile comes
  // from HBM about once and from L2 after that (all heads of one row block at once
  // would stream every tile from HBM once per row block). Within a head the
  // heaviest row blocks (most key tiles) go first.
  const int64_t bh = blockIdx.x / p.row_blocks;
  const int rb = p.row_blocks - 1 - (int)(blockIdx.x % p.row_blocks);
  const int b = (int)(bh / kMhaHeads), h = (int)(bh % kMhaHeads);
  const int i0 = rb * kMhaTile;  // first window row of the block
  const SeqRows R = seq_rows(p.q_start, p.seqlens, b, p.q_per_seq, p.num_q, p.max_ctx);
  const bool seq_ok = R.ok;
  // window rows of this block that the sequence has (a ragged batch's shorter
  // sequences have fewer than the window)
  const int rows_here = min(p.row_count, R.q_len - p.row_begin);
  const int last_i = min(i0 + kMhaTile, rows_here) - 1;
  const int pos_last = R.seqlen - R.q_len + p.row_begin + last_i;
  const int nt = (seq_ok && last_i >= i0 && pos_last >= 0) ? pos_last / kMhaTile + 1 : 0;

  if (tid == 0) {
    mbar_init(smem_u32(qfull), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&kfull[i]), 1);
      mbar_init(smem_u32(&kempty[i]), 1);
      mbar_init(smem_u32(&vfull[i]), 1);
      mbar_init(smem_u32(&vempty[i]), 1);
      mbar_init(smem_u32(&sfull[i]), 1);
      mbar_init(smem_u32(&pfull[i]), 128);
    }
    mbar_init(smem_u32(odone), 1);
    mbar_init(smem_u32(mdone), 1);
    *abort_flag = 0;
    fence_mbarrier_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint64_t TO = p.timeout_ns;
  int drain_dummy = 0;
  volatile int* no_abort = &drain_dummy;
  const int64_t kv_row0 = ((int64_t)b * kMhaHeads + h) * p.ctx_pad;  // this head's keys
  const int64_t kr_row0 = (int64_t)b * p.ctx_pad;

  if (warp == 0 || warp == 6) {
    // ------------------------------------------------------------ TMA producers
    // warp 0: Q once, then the key tiles; warp 6: the value tiles
    const bool keys = warp == 0;
    int issued = 0;
    if (lane == 0 && nt > 0) {
      bool ok = true;
      if (keys) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_kn);
        prefetch_tmap(&tm_kr);
        const int t0 = (int)(R.t0 + p.row_begin + i0);
        const uint32_t bar = smem_u32(qfull);
        mbar_arrive_expect_tx(bar, kFaQBytes);
        for (int c = 0; c < 3; ++c) tma_load_3d(smem_u32(sQ + c * kFaQChunk), &tm_q, bar, 64 * c, h, t0);
      } else {
        prefetch_tmap(&tm_v);
      }
      for (int j = 0; ok && j < nt; ++j) {
        const int st = j & 1;
        if (keys) {
          ok = mbar_wait(smem_u32(&kempty[st]), ((j >> 1) & 1) ^ 1, TO, abort_flag);
          if (!ok) break;
          const uint32_t bar = smem_u32(&kfull[st]);
          const uint32_t dst = smem_u32(sK + st * kFaKBytes);
          mbar_arrive_expect_tx(bar, kFaKBytes);
          tma_load_2d(dst, &tm_kn, bar, 0, (int)(kv_row0 + j * kMhaTile));
          tma_load_2d(dst + kFaQChunk, &tm_kn, bar, 64, (int)(kv_row0 + j * kMhaTile));
          tma_load_2d(dst + 2 * kFaQChunk, &tm_kr, bar, 0, (int)(kr_row0 + j * kMhaTile));
        } else {
          ok = mbar_wait(smem_u32(&vempty[st]), ((j >> 1) & 1) ^ 1, TO, abort_flag);
          if (!ok) break;
          const uint32_t bar = smem_u32(&vfull[st]);
          const uint32_t dst = smem_u32(sV + st * kFaVBytes);
          mbar_arrive_expect_tx(bar, kFaVBytes);
          tma_load_2d(dst, &tm_v, bar, 0, (int)(kv_row0 + j * kMhaTile));
          tma_load_2d(dst + kFaQChunk, &tm_v, bar, 64, (int)(kv_row0 + j * kMhaTile));
        }
        issued = j + 1;
      }
      // on an early exit, let the copies still in flight land before the CTA can leave
      if (keys) mbar_wait(smem_u32(qfull), 0, TO, no_abort);
      for (int j = issued > 2 ? issued - 2 : 0; j < issued; ++j)
        mbar_wait(smem_u32(keys ? &kfull[j & 1] : &vfull[j & 1]), (j >> 1) & 1, TO, no_abort);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Issue order S_0, S_1, then P_j.V followed by S_{j+2}, which reuses the score
    // buffer that P_j.V reads (the tensor core runs one CTA's MMAs in order).
    if (lane == 0 && nt > 0) {
      const uint32_t idesc_s = instr_desc(1 /*bf16*/, 0, 0, 128, kMhaTile);
      const uint32_t idesc_pv = instr_desc(1, 0, 1 /*V is MN-major*/, 128, kMhaDv);
      bool ok = mbar_wait(smem_u32(qfull), 0, TO, abort_flag);
      auto issue_s = [&](int j) {  // S_j = Q . K_j^T, K = 128 nope + 64 rope dims
        const int st = j & 1;
        tc_fence_after();
        const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK + st * kFaKBytes);
#pragma unroll
        for (int kk = 0; kk < kMhaDqk / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kFaQChunk + (kk & 3) * 32;
          mma_bf16_ss(tmem_base + st * kMhaTile, smem_desc_sw128(qa + off, 16, 1024),
                      smem_desc_sw128(ka + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&sfull[st]));
        mma_commit(smem_u32(&kempty[st]));
      };
      for (int j = 0; ok && j < 2 && j < nt; ++j) {
        ok = mbar_wait(smem_u32(&kfull[j]), 0, TO, abort_flag);
        if (ok) issue_s(j);
      }
      for (int j = 0; ok && j < nt; ++j) {
        const int st = j & 1;
        ok = mbar_wait(smem_u32(&pfull[st]), (j >> 1) & 1, TO, abort_flag) &&
             mbar_wait(smem_u32(&vfull[st]), (j >> 1) & 1, TO, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t va = smem_u32(sV + st * kFaVBytes);
#pragma unroll
        for (int kk = 0; kk < kMhaTile / 16; ++kk)  // P from TMEM: 16 keys = 8 columns
          mma_bf16_ts(tmem_base + kFaTmemO, tmem_base + st * kMhaTile + kk * 8,
                      smem_desc_sw128(va + kk * 2048, kFaQChunk, 1024), idesc_pv,
                      (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(smem_u32(&vempty[st]));
        mma_commit(smem_u32(odone));
        if (j + 2 < nt) {
          ok = mbar_wait(smem_u32(&kfull[st]), ((j + 2) >> 1) & 1, TO, abort_flag);
          if (ok) issue_s(j + 2);
        }
      }
      mma_commit(smem_u32(mdone));
      mbar_wait(smem_u32(mdone), 0, TO, no_abort);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    // thread = query row (TMEM lane); warps 2-5 cover lane quadrants 2, 3, 0, 1
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tO = tmem_base + kFaTmemO + lane_off;
    const int i = i0 + r;  // window row
    const bool row_ok = seq_ok && i < rows_here;
    const int qi = p.row_begin + i;
    const int pos = row_ok ? R.seqlen - R.q_len + qi : -1;  // -1: sees no key
    const int64_t t = R.t0 + qi;
    const bool use_mask = p.mask != nullptr && row_ok && pos + 1 > p.k;
    const uint4* mrow =
        use_mask ? reinterpret_cast<const uint4*>(p.mask + t * p.mask_ld) : nullptr;
    const uint4 all_bits = make_uint4(~0u, ~0u, ~0u, ~0u);
    uint4 mw = (use_mask && nt > 0) ? __ldg(mrow) : all_bits;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; ok && j < nt; ++j) {
      const int st = j & 1;
      const int kbase = j * kMhaTile;
      const uint4 mw_next =
          (use_mask && j + 1 < nt && kbase + kMhaTile <= pos) ? __ldg(mrow + j + 1) : all_bits;
      ok = warp_wait(smem_u32(&sfull[st]), (j >> 1) & 1, TO, abort_flag);
      if (!ok) break;
      tc_fence_after();
      uint32_t x[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32u(tmem_base + st * kMhaTile + c * 32 + lane_off, x[c]);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_wait_ld_fence(x[c]);
      // Keys outside the row's set become -inf. One 32-bit validity word per
      // 32-key chunk (causal limit AND selection bits); the running max of the raw
      // scores uses four independent accumulators (a single warp per SM
      // sub-partition runs each row, so dependent chains, not issue, set its pace).
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t bits = c == 0 ? mw.x : c == 1 ? mw.y : c == 2 ? mw.z : mw.w;
        const int lim = pos - kbase - 32 * c;  // last visible key of the chunk
        const uint32_t vm =
            bits & (lim >= 31 ? 0xffffffffu : (lim < 0 ? 0u : (2u << lim) - 1u));
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float v = ((vm >> e) & 1u) ? __uint_as_float(x[c][e]) : -INFINITY;
          x[c][e] = __float_as_uint(v);
          mx[e & 3] = fmaxf(mx[e & 3], v);
        }
      }
      // tile max in base-2 logits (the scale is positive)
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
      // lazy rescale: the reference max moves only when it grows by more than 8
      const bool grow = m_ref != -INFINITY && mt > m_ref + 8.f;
      if (__any_sync(0xffffffffu, grow)) {
        // O holds P.V of the tiles before j (j >= 1 here): wait for the last one.
        // S_j completed after P_{j-2}.V (issue order), so at most P_{j-1}.V is
        // open and the parity of odone identifies it.
        ok = warp_wait(smem_u32(odone), (j - 1) & 1, TO, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const float f = grow ? exp2f(m_ref - mt) : 1.f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= f;
          tmem_st32(tO + c * 32, o);
        }
        tmem_wait_st();
        if (grow) {
          l *= f;
          m_ref = mt;
        }
      }
      if (m_ref == -INFINITY) m_ref = mt;  // first visible key (stays -inf without one)
      // P = 2^(z - m_ref), rounded to bf16 for the MMA, written over the first 64
      // columns of the scores
      // p = 2^(s * scale_log2 - m_ref) as one FFMA and one ex2 per key (-inf -> 0)
      const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
      const float s2 = p.scale_log2;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        float pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = (64 * h2 + 2 * e) >> 5, w = (64 * h2 + 2 * e) & 31;
          const float p0 = ex2_approx(fmaf(__uint_as_float(x[c][w]), s2, neg_m));
          const float p1 = ex2_approx(fmaf(__uint_as_float(x[c][w + 1]), s2, neg_m));
          ls[e & 3] += p0 + p1;  // the softmax sum from the unrounded values (exact LSE)
          pk[e] = __uint_as_float(pack_bf16x2(p0, p1));
        }
        tmem_st32(tmem_base + st * kMhaTile + h2 * 32 + lane_off, pk);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&pfull[st]));
      mw = mw_next;
    }
    // every MMA done (the last P.V included): the one-shot barrier the MMA warp
    // commits at its end (a parity wait on odone could pass while two P.V are open)
    if (ok && nt > 0) ok = warp_wait(smem_u32(mdone), 0, TO, abort_flag);
    tc_fence_after();
    __nv_bfloat16* orow = p.out + (t * kMhaHeads + h) * kMhaDv;
    const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float o[32];
      if (ok && nt > 0) {
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
      }
      if (row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 v4 = make_uint4(0, 0, 0, 0);
          if (ok && nt > 0 && l > 0.f)
            v4 = make_uint4(pack_bf16x2(o[8 * q] * inv, o[8 * q + 1] * inv),
                            pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                            pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                            pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
          dst[q] = v4;
        }
      }
    }
    if (row_ok)
      p.lse[t * kMhaHeads + h] =
          l > 0.f ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
    if (!seq_ok && r == 0 && h == 0 && rb == 0) report_error(kErrBounds);
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace dsa
