// indexer_kl.cuh -- the lightning indexer's training target and KL loss term on
// the sm_100a tensor cores.
//
// DeepSeek-V3.2-Exp technical report (zh translation), §2.1: the main attention
// of token t, summed over all heads and L1-normalised along the sequence, is the
// target distribution p_{t,:}; the indexer is trained with the KL divergence
// between p_{t,:} and Softmax(I_{t,:}) — over every visible key in the dense
// warm-up stage, over the selected set S_t in the sparse stage. With the main
// attention a_h(s) = softmax_{s in S}(scale q_h . c_s) of each head,
//   p(s) = mean_h a_h(s),  q(s) = softmax_{s in S}(I_{t,s}),
//   KL_t = sum_s p(s) (ln p(s) - ln q(s))
//        = sum_s p ln p - sum_s p I_s + (sum_s p) lse_I,  lse_I = ln sum_s e^{I_s}.
// a_h(s) = exp(scale q_h . c_s - LSE_h) uses the forward's per-head LSE.
//
// One CTA per query token, no cluster and no O accumulator: the 128 heads of a
// key are the N side of one MMA. Per tile of 128 listed keys the tensor core
// computes D[key][head] = K_tile (128 x 576) . Q^T (576 x 128) into one of two
// TMEM accumulators (M = 128 keys, N = 128 heads, K = 576 as 9 chunks x 4
// K-steps); Q stays in shared memory for the whole token (9 swizzled 64-dim
// chunks), the keys' latent rows stream through a 5-stage ring of 64-dim chunks.
//
// Warp roles (288 threads):
//   warps 0-3   epilogue, thread = key lane: 128 heads' exp2 per key, the head
//               mean p, and running sums of p ln p, p I, p and a log-sum-exp of I
//   warp 4      TMEM allocation + single-thread MMA issue
//   warps 5-8   producers: Q into shared memory, then per tile each thread
//               resolves one listed key (-1 outside [0, pos]: zero row, p = 0)
//               and copies its 9 x 128 B with cp.async (zero fill when invalid)
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "rows.cuh"

namespace dsa {

constexpr int kKlHeads = 128;
constexpr int kKlDqk = 576;
constexpr int kKlChunks = kKlDqk / 64;             // 9 chunks of 64 dims (128 B)
constexpr int kKlTile = 128;                       // keys per tile (MMA M)
constexpr int kKlStages = 5;
constexpr int kKlThreads = 288;
constexpr int kKlChunkBytes = 128 * 128;           // 128 rows x 128 B
constexpr int kKlSmemBytes = 1024 + kKlChunks * kKlChunkBytes /*Q*/ +
                             kKlStages * kKlChunkBytes /*keys*/ + kKlHeads * 4 /*lse2*/ +
                             2 * kKlTile * 4 /*listed positions*/ + 4 * 8 * 4 /*reduction*/ +
                             24 * 8 /*barriers*/ + 16;
static_assert(kKlSmemBytes <= 232448, "indexer KL shared memory exceeds the per-CTA limit");

struct KlParams {
  const uint8_t* kv;           // latent cache rows of 1152 B
  const __nv_bfloat16* q;      // [T][128][576]
  const int32_t* idx;          // [T][k]
  const float* lse;            // [T][128] natural-log LSE of the forward
  const float* scores;         // [batch * row_count][ld] indexer score rows of the window
  const int32_t* block_table;  // paged
  const int32_t* seqlens;      // [batch] or nullptr
  float* kl;                   // [batch * row_count]
  int64_t ld;
  int32_t k, batch, max_ctx, q_per_seq;
  int32_t row_begin, row_count;
  int32_t paged, page_size, max_pages, num_pages;
  float scale_log2;            // scale * log2(e)
  uint64_t timeout_ns;
  const int32_t* q_start;      // [batch + 1] ragged query rows, or nullptr (rows.cuh)
  int32_t num_q;
};

__global__ void __launch_bounds__(kKlThreads, 1) indexer_kl_kernel(const __grid_constant__ KlParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                                         // [9][128][128 B] swizzled
  uint8_t* sK = sQ + kKlChunks * kKlChunkBytes;               // [4][128][128 B] swizzled
  float* sLse2 = reinterpret_cast<float*>(sK + kKlStages * kKlChunkBytes);  // [128] LSE*log2e
  int32_t* sSel = reinterpret_cast<int32_t*>(sLse2 + kKlHeads);  // [2][128] positions (-1: none)
  float* sRed = reinterpret_cast<float*>(sSel + 2 * kKlTile);              // [4 warps][8]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRed + 32);
  uint64_t* kfull = bars;                    // [4] chunk landed (128 producer arrivals)
  uint64_t* kempty = kfull + kKlStages;      // [4] MMA read the chunk
  uint64_t* tfull = kempty + kKlStages;      // [2] accumulator ready
  uint64_t* tempty = tfull + 2;              // [2] epilogue done with it (128)
  uint64_t* qfull = tempty + 2;              // Q and the LSE row stored (128)
  uint64_t* sready = qfull + 1;              // [2] producers wrote the tile's positions (128)
  uint64_t* rfree = sready + 2;              // [2] epilogue read them (128)
  uint64_t* mdone = rfree + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mdone + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t local = blockIdx.x;                       // row of the window
  const int b = (int)(local / p.row_count);
  const int qi = p.row_begin + (int)(local - (int64_t)b * p.row_count);
  const SeqRows R = seq_rows(p.q_start, p.seqlens, b, p.q_per_seq, p.num_q, p.max_ctx);
  if (qi >= R.q_len) {  // a window row the sequence does not have (ragged batch): no term
    if (tid == 0) {
      if (!R.ok) report_error(kErrBounds);
      p.kl[local] = 0.f;
    }
    return;
  }
  const int64_t t = R.t0 + qi;                            // global query row
  const int ntiles = (p.k + kKlTile - 1) / kKlTile;
  const bool seq_ok = R.ok;
  const int pos = R.seqlen - R.q_len + qi;

  if (tid == 0) {
    for (int i = 0; i < kKlStages; ++i) {
      mbar_init(smem_u32(&kfull[i]), 128);
      mbar_init(smem_u32(&kempty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), 128);
      mbar_init(smem_u32(&sready[i]), 128);
      mbar_init(smem_u32(&rfree[i]), 128);
    }
    mbar_init(smem_u32(qfull), 128);
    mbar_init(smem_u32(mdone), 1);
    *abort_flag = 0;
    fence_mbarrier_init_cluster();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_holder), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint64_t TO = p.timeout_ns;
  int drain_dummy = 0;
  volatile int* no_abort = &drain_dummy;

  if (warp >= 5) {
    // ------------------------------------------------------------ producers
    const int pt = tid - 160;  // 0..127
    {
      // Q row h = pt: 9 chunks of 128 B, 16-B pieces at their swizzled places
      const uint4* src = reinterpret_cast<const uint4*>(p.q + (t * kKlHeads + pt) * kKlDqk);
#pragma unroll 1
      for (int c = 0; c < kKlChunks; ++c) {
        uint4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __ldg(src + c * 8 + i);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<uint4*>(sQ + c * kKlChunkBytes + sw128_offset(pt, i)) = v[i];
      }
      sLse2[pt] = __ldg(p.lse + t * kKlHeads + pt) * 1.4426950408889634f;
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(qfull));
    }
    uint32_t it = 0;  // chunk counter over all tiles
    bool ok = true;
    // This thread's key of tile T is entry T*128 + pt of the row's list. Its
    // position is loaded two tiles ahead and its page one tile ahead, so no
    // tile waits on those dependent loads.
    auto load_sel = [&](int tile) -> int {
      const int e = tile * kKlTile + pt;
      int sel = (tile < ntiles && e < p.k) ? __ldg(p.idx + t * p.k + e) : -1;
      return (seq_ok && sel >= 0 && sel <= pos) ? sel : -1;
    };
    auto load_page = [&](int sel) -> int {
      return (p.paged && sel >= 0) ? __ldg(p.block_table + (int64_t)b * p.max_pages + sel / p.page_size)
                                   : 0;
    };
    int sel_a = load_sel(0), sel_b = load_sel(1);
    int pg_a = load_page(sel_a);
    for (int tile = 0; tile < ntiles && ok; ++tile) {
      int sel = sel_a;
      const int pg = pg_a;
      pg_a = load_page(sel_b);
      sel_a = sel_b;
      sel_b = load_sel(tile + 2);
      int64_t row = -1;
      if (sel >= 0) {
        if (!p.paged) {
          row = (int64_t)b * p.max_ctx + sel;
        } else if (pg >= 0 && pg < p.num_pages) {
          row = (int64_t)pg * p.page_size + sel % p.page_size;
        } else {
          report_error(kErrBounds);
          sel = -1;
        }
      }
      // positions slot tile & 1: its previous tile (two back) must have been read
      if (tile >= 2)
        ok = warp_wait(smem_u32(&rfree[tile & 1]), ((tile >> 1) - 1) & 1, TO, abort_flag);
      if (!ok) break;
      sSel[(tile & 1) * kKlTile + pt] = sel;
      mbar_arrive(smem_u32(&sready[tile & 1]));
      const uint8_t* src = p.kv + (row >= 0 ? row * (kKlDqk * 2) : 0);
#pragma unroll 1
      for (int c = 0; c < kKlChunks; ++c, ++it) {
        const int st = it % kKlStages;
        if (!warp_wait(smem_u32(&kempty[st]), ((it / kKlStages) & 1) ^ 1, TO, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t dst = smem_u32(sK + st * kKlChunkBytes);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          cp_async_16(dst + sw128_offset(pt, i), src + c * 128 + i * 16, row >= 0 ? 16u : 0u);
        cp_async_mbar_arrive(smem_u32(&kfull[st]));
      }
    }
    cp_async_wait_all();
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = instr_desc(1 /*bf16*/, 0, 0, 128, 128);
      uint32_t it = 0;
      bool ok = mbar_wait(smem_u32(qfull), 0, TO, abort_flag);
      if (ok) tc_fence_after();
      for (int tile = 0; tile < ntiles && ok; ++tile) {
        const int ab = tile & 1;
        if (!mbar_wait(smem_u32(&tempty[ab]), ((tile >> 1) & 1) ^ 1, TO, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + ab * 128;
        for (int c = 0; c < kKlChunks; ++c, ++it) {
          const int st = it % kKlStages;
          if (!mbar_wait(smem_u32(&kfull[st]), (it / kKlStages) & 1, TO, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          fence_proxy_async_smem();  // cp.async (generic proxy) writes -> tensor-core reads
          const uint32_t ka = smem_u32(sK + st * kKlChunkBytes);
          const uint32_t qa = smem_u32(sQ + c * kKlChunkBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(d, smem_desc_sw128(ka + kk * 32, 16, 1024),
                        smem_desc_sw128(qa + kk * 32, 16, 1024), idesc, (c > 0 || kk > 0) ? 1u : 0u);
          mma_commit(smem_u32(&kempty[st]));
        }
        if (ok) mma_commit(smem_u32(&tfull[ab]));
      }
      mma_commit(smem_u32(mdone));
      mbar_wait(smem_u32(mdone), 0, TO, no_abort);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int e_lane = warp * 32 + lane;                 // key lane == TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float* srow = p.scores + local * p.ld;
    float s_plnp = 0.f, s_pi = 0.f, s_p = 0.f;         // sums over this thread's keys
    float m_i = -INFINITY, s_i = 0.f;                  // running log-sum-exp of I (base e)
    bool ok = mbar_wait(smem_u32(qfull), 0, TO, abort_flag);
    for (int tile = 0; tile < ntiles && ok; ++tile) {
      const int ab = tile & 1;
      ok = warp_wait(smem_u32(&tfull[ab]), (tile >> 1) & 1, TO, abort_flag);
      if (ok) ok = warp_wait(smem_u32(&sready[tile & 1]), (tile >> 1) & 1, TO, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const int sel = sSel[(tile & 1) * kKlTile + e_lane];
      // p(s) = mean over heads of exp(z_h - LSE_h), in base 2
      float psum = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float z[32];
        tmem_ld32(tmem_base + ab * 128 + c * 32 + lane_off, z);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) psum += ex2_approx(z[i] * p.scale_log2 - sLse2[c * 32 + i]);
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&tempty[ab]));
      if (sel >= 0) {
        const float pv = psum * (1.0f / kKlHeads);
        const float iv = __ldg(srow + sel);
        if (pv > 0.f) s_plnp += pv * logf(pv);
        s_pi += pv * iv;
        s_p += pv;
        if (iv > m_i) {
          s_i = s_i * expf(m_i - iv) + 1.0f;
          m_i = iv;
        } else {
          s_i += expf(iv - m_i);
        }
      }
      mbar_arrive(smem_u32(&rfree[tile & 1]));
    }
    // block reduction over the 128 keys lanes: sums and the log-sum-exp
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s_plnp += __shfl_xor_sync(0xffffffffu, s_plnp, o);
      s_pi += __shfl_xor_sync(0xffffffffu, s_pi, o);
      s_p += __shfl_xor_sync(0xffffffffu, s_p, o);
      const float m2 = __shfl_xor_sync(0xffffffffu, m_i, o);
      const float s2 = __shfl_xor_sync(0xffffffffu, s_i, o);
      const float m = fmaxf(m_i, m2);
      s_i = (m == -INFINITY) ? 0.f : s_i * expf(m_i - m) + s2 * expf(m2 - m);
      m_i = m;
    }
    const bool all_ok = named_barrier_and(1, 128, ok);
    if (lane == 0) {
      sRed[warp * 8 + 0] = s_plnp;
      sRed[warp * 8 + 1] = s_pi;
      sRed[warp * 8 + 2] = s_p;
      sRed[warp * 8 + 3] = m_i;
      sRed[warp * 8 + 4] = s_i;
    }
    named_barrier_sync(1, 128);
    if (tid == 0 && all_ok) {
      float a = 0.f, bpi = 0.f, ps = 0.f, m = -INFINITY, s = 0.f;
      for (int w = 0; w < 4; ++w) {
        a += sRed[w * 8 + 0];
        bpi += sRed[w * 8 + 1];
        ps += sRed[w * 8 + 2];
        const float m2 = sRed[w * 8 + 3], s2 = sRed[w * 8 + 4];
        const float mm = fmaxf(m, m2);
        s = (mm == -INFINITY) ? 0.f : s * expf(m - mm) + s2 * expf(m2 - mm);
        m = mm;
      }
      const float lse_i = s > 0.f ? m + logf(s) : 0.f;
      p.kl[local] = ps > 0.f ? a - bpi + ps * lse_i : 0.f;
    }
    if (tid == 0 && !seq_ok) report_error(kErrBounds);
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

}  // namespace dsa
