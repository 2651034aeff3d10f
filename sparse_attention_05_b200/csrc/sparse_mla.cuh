// sparse_mla.cuh -- sparse MLA forward in MQA mode on the sm_100a tensor cores.
//
// DeepSeek-V3.2-Exp technical report (zh translation), §1 "Architecture",
// Eq. 2 and Fig. 1: u_t = Attn(h_t, {c_s : s in S_t}), DSA instantiated on MLA
// in MQA mode, i.e. every one of the 128 query heads of token t attends over
// the SAME selected latent rows c_s (576-d key = 512 latent + 64 rope; the value
// is the 512-d latent). Per head h:
//   z_s = scale * q_{t,h} . c_s,  LSE_h = ln sum_s exp(z_s),  o_h = sum_s e^{z_s - LSE_h} c_s[0:512].
//
// Design: one 2-CTA cluster per query token. O (128 heads x 512 fp32) would
// fill all of one SM's tensor memory, so CTA r of the pair owns value dims
// [256 r, 256 r + 256) and contracts QK^T over its own slice of the key dims:
//   r = 0: key dims [0, 256)    (= its value dims)
//   r = 1: key dims [256, 576)  (its value dims + the 64 rope dims)
// Every gathered latent byte is loaded by exactly one CTA. The two partial
// score tiles S_r = Q[:, slice_r] . K[:, slice_r]^T are swapped through
// distributed shared memory and added (a + b == b + a, so both CTAs hold
// bit-identical S and take identical softmax decisions); then each CTA runs
// O_r += P . V[:, value dims of r] on its own half.
//
// Per 64-key block j (double-buffered):
//   producers (warps 0-3)  gather the block's rows (their slice) with cp.async
//                          into the canonical 128-B-swizzled layout, zero-filling
//                          entries outside [0, pos(t)]
//   MMA (warp 8, 1 thread) S_j = Q . K_j^T  (M=128 heads, N=64 keys, K=256|320)
//                          then O += P_{j-1} . V_{j-1} (M=128, N=256, K=64, V MN-major)
//   softmax (warps 4-7)    thread = head: S from TMEM, partial swap with the
//                          peer CTA, online softmax in base 2 with a lazy
//                          rescale of O (only when the running max grows by
//                          more than 2^8), P as bf16 into shared memory
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dsa {

constexpr int kMlaHeads = 128;
constexpr int kMlaDqk = 576;
constexpr int kMlaDv = 512;
constexpr int kMlaBlk = 64;                  // keys per block
constexpr int kMlaThreads = 288;             // 4 producer warps, 4 softmax warps, 1 MMA warp
constexpr int kMlaQChunk = kMlaHeads * 128;  // one 64-dim column chunk of Q: 16 KB
constexpr int kMlaKChunk = kMlaBlk * 128;    // one 64-dim column chunk of a key block: 8 KB
constexpr int kMlaStageBytes = 5 * kMlaKChunk;  // up to 320 dims per CTA
constexpr int kMlaPBytes = kMlaHeads * 128;     // 128 heads x 64 keys bf16
constexpr int kMlaXBytes = kMlaHeads * kMlaBlk * 4;
constexpr int kMlaSmemBytes = 1024 + 5 * kMlaQChunk + 2 * kMlaStageBytes + 2 * kMlaPBytes +
                              kMlaXBytes + 2 * kMlaBlk * 4 /*rows*/ + 2 * 8 /*masks*/ +
                              32 * 8 /*barriers*/ + 16;
constexpr uint32_t kMlaTmemCols = 512;       // O: [0,256), S buffers: [256,320), [320,384)

struct MlaParams {
  const uint8_t* kv;           // latent cache rows of 1152 B
  const int32_t* idx;          // [T][k]
  const int32_t* block_table;  // paged
  const int32_t* seqlens;      // [batch] or nullptr
  __nv_bfloat16* out;          // [T][128][512]
  float* lse;                  // [T][128]
  int32_t k, batch, max_ctx, q_per_seq;
  int32_t paged, page_size, max_pages, num_pages;
  int64_t cache_rows;
  float scale_log2;            // scale * log2(e)
  uint64_t timeout_ns;
};

__global__ void __launch_bounds__(kMlaThreads, 1)
    sparse_mla_kernel(const __grid_constant__ MlaParams p, const __grid_constant__ CUtensorMap tm_q) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + 5 * kMlaQChunk;
  uint8_t* sP = sKV + 2 * kMlaStageBytes;
  uint8_t* sX = sP + 2 * kMlaPBytes;
  int32_t* sRow = reinterpret_cast<int32_t*>(sX + kMlaXBytes);   // [2][64] cache rows, -1 = skip
  uint64_t* sMask = reinterpret_cast<uint64_t*>(sRow + 2 * kMlaBlk);  // [2] valid-key masks
  uint64_t* bars = sMask + 2;
  uint64_t* kvfull = bars + 0;   // [2]
  uint64_t* kvempty = bars + 2;  // [2]
  uint64_t* sfull = bars + 4;    // [2]
  uint64_t* sfree = bars + 6;    // [2]
  uint64_t* pfull = bars + 8;    // [2]
  uint64_t* qfull = bars + 10;
  uint64_t* ofull = bars + 11;
  uint64_t* xfull = bars + 12;
  uint64_t* xfree = bars + 13;
  uint64_t* mdone = bars + 14;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int64_t t = blockIdx.x >> 1;
  const int b = (int)(t / p.q_per_seq);
  const int nchunk = 4 + (int)rank;      // 64-dim column chunks of this CTA's key slice
  const int d0 = 256 * (int)rank;        // first key dim of the slice (also first value dim)
  const int nblk = (p.k + kMlaBlk - 1) / kMlaBlk;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&kvfull[i]), 128);
      mbar_init(smem_u32(&kvempty[i]), 1);
      mbar_init(smem_u32(&sfull[i]), 1);
      mbar_init(smem_u32(&sfree[i]), 128);
      mbar_init(smem_u32(&pfull[i]), 128);
    }
    mbar_init(smem_u32(qfull), 1);
    mbar_init(smem_u32(ofull), 1);
    mbar_init(smem_u32(xfull), 128);
    mbar_init(smem_u32(xfree), 128);
    mbar_init(smem_u32(mdone), 1);
    *abort_flag = 0;
    fence_mbarrier_init_cluster();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_holder), kMlaTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  // Both CTAs' barriers must be initialised before the peer may touch them.
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t tO = tmem_base, tS0 = tmem_base + 256;
  const uint64_t TO = p.timeout_ns;
  int drain_dummy = 0;
  volatile int* no_abort = &drain_dummy;

  // Position of this query row and validity of its sequence.
  const int seqlen = p.seqlens ? __ldg(p.seqlens + b) : p.max_ctx;
  const bool seq_ok = seqlen >= p.q_per_seq && seqlen <= p.max_ctx;
  const int pos = seqlen - p.q_per_seq + (int)(t % p.q_per_seq);

  if (warp < 4) {
    // ------------------------------------------------------------ gather producers
    const int nch16 = nchunk * 8;  // 16-byte chunks per row slice
    for (int j = 0; j < nblk; ++j) {
      const int st = j & 1;
      // the stage is free once O += P V of block j-2 has finished; the four
      // producer warps take this decision together (no warp is left behind
      // in a barrier when a wait gives up)
      const bool ok = warp_wait(smem_u32(&kvempty[st]), ((j >> 1) & 1) ^ 1, TO, abort_flag);
      if (!named_barrier_and(1, 128, ok)) break;
      if (tid < kMlaBlk) {
        const int e = j * kMlaBlk + tid;
        const int s = e < p.k ? __ldg(p.idx + t * p.k + e) : -1;
        int row = -1;
        if (seq_ok && s >= 0 && s <= pos) {
          if (!p.paged) {
            row = b * p.max_ctx + s;
          } else {
            const int pg = __ldg(p.block_table + (int64_t)b * p.max_pages + s / p.page_size);
            if (pg >= 0 && pg < p.num_pages) row = pg * p.page_size + s % p.page_size;
            else report_error(kErrBounds);
          }
        }
        sRow[st * kMlaBlk + tid] = row;
        const uint32_t m = __ballot_sync(0xffffffffu, row >= 0);
        if (lane == 0) reinterpret_cast<uint32_t*>(&sMask[st])[warp] = m;
      }
      named_barrier_sync(1, 128);
      const uint32_t stage = smem_u32(sKV + st * kMlaStageBytes);
      for (int ci = tid; ci < kMlaBlk * nch16; ci += 128) {
        const int kr = ci / nch16, c = ci - kr * nch16;
        const int row = sRow[st * kMlaBlk + kr];
        const uint8_t* src = p.kv + (row >= 0 ? (int64_t)row * (kMlaDqk * 2) : 0) + d0 * 2 + c * 16;
        cp_async_16(stage + (c >> 3) * kMlaKChunk + sw128_offset(kr, c & 7), src,
                    row >= 0 ? 16u : 0u);
      }
      cp_async_commit();
      // Only one block can be in flight (two stages: one loading, one in use),
      // so wait for this block and publish it right away.
      cp_async_wait_group<0>();
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&kvfull[st]));
    }
    cp_async_wait_group<0>();
    __syncwarp();
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool q_seen = false;
      const uint32_t qb = smem_u32(qfull);
      mbar_arrive_expect_tx(qb, nchunk * kMlaQChunk);
      for (int c = 0; c < nchunk; ++c)
        tma_load_2d(smem_u32(sQ + c * kMlaQChunk), &tm_q, qb, d0 + 64 * c, (int)(t * kMlaHeads));
      const uint32_t idesc_s = instr_desc(1 /*bf16*/, 0, 0, 128, kMlaBlk);
      const uint32_t idesc_pv = instr_desc(1, 0, 1 /*V is MN-major*/, 128, 256);
      auto pv = [&](int j) -> bool {
        if (!mbar_wait(smem_u32(&pfull[j & 1]), (j >> 1) & 1, TO, abort_flag)) return false;
        tc_fence_after();
        const uint32_t pa = smem_u32(sP + (j & 1) * kMlaPBytes);
        const uint32_t va = smem_u32(sKV + (j & 1) * kMlaStageBytes);
#pragma unroll
        for (int kk = 0; kk < kMlaBlk / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(pa + kk * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(va + kk * 2048, kMlaKChunk, 1024);
          mma_bf16_ss(tO, ad, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(smem_u32(&kvempty[j & 1]));
        mma_commit(smem_u32(ofull));
        return true;
      };
      if (mbar_wait(qb, 0, TO, abort_flag)) {
        q_seen = true;
        for (int j = 0; j < nblk; ++j) {
          const int st = j & 1;
          if (!mbar_wait(smem_u32(&kvfull[st]), (j >> 1) & 1, TO, abort_flag) ||
              !mbar_wait(smem_u32(&sfree[st]), ((j >> 1) & 1) ^ 1, TO, abort_flag))
            break;
          tc_fence_after();
          const uint32_t ka = smem_u32(sKV + st * kMlaStageBytes);
          const uint32_t qa = smem_u32(sQ);
          for (int kk = 0; kk < nchunk * 4; ++kk) {
            const uint64_t ad = smem_desc_sw128(qa + (kk >> 2) * kMlaQChunk + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(ka + (kk >> 2) * kMlaKChunk + (kk & 3) * 32, 16, 1024);
            mma_bf16_ss(tS0 + st * kMlaBlk, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&sfull[st]));
          if (j > 0 && !pv(j - 1)) break;
          if (j == nblk - 1) pv(j);
        }
      }
      if (!q_seen) mbar_wait(qb, 0, TO, no_abort);  // the Q load must land before exit
      mma_commit(smem_u32(mdone));
      mbar_wait(smem_u32(mdone), 0, TO, no_abort);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int h = tid - 128;  // head == TMEM lane
    const int quad = warp - 4;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t x_local = smem_u32(sX);
    const uint32_t x_peer = mapa_shared(x_local, peer);
    const uint32_t xfull_peer = mapa_shared(smem_u32(xfull), peer);
    const uint32_t xfree_peer = mapa_shared(smem_u32(xfree), peer);
    const uint32_t prow = (uint32_t)h * 1024u / 8u;  // h * 128
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk && ok; ++j) {
      const int st = j & 1;
      float s[64];
      if (!warp_wait(smem_u32(&sfull[st]), (j >> 1) & 1, TO, abort_flag)) { ok = false; break; }
      tc_fence_after();
      {
        float a[32], c[32];
        tmem_ld32(tS0 + st * kMlaBlk + lane_off, a);
        tmem_ld32(tS0 + st * kMlaBlk + 32 + lane_off, c);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = a[i];
          s[32 + i] = c[i];
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&sfree[st]));
      // swap partial scores with the peer CTA
      if (j > 0 && !warp_wait<true>(smem_u32(xfree), (j - 1) & 1, TO, abort_flag)) { ok = false; break; }
#pragma unroll
      for (int c = 0; c < 16; ++c)
        st_cluster_v4(x_peer + h * 256 + ((c ^ (h & 7)) << 4), s[4 * c], s[4 * c + 1],
                      s[4 * c + 2], s[4 * c + 3]);
      mbar_arrive_remote(xfull_peer);
      if (!warp_wait<true>(smem_u32(xfull), j & 1, TO, abort_flag)) { ok = false; break; }
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 v = *reinterpret_cast<const float4*>(sX + h * 256 + ((c ^ (h & 7)) << 4));
        s[4 * c] += v.x;
        s[4 * c + 1] += v.y;
        s[4 * c + 2] += v.z;
        s[4 * c + 3] += v.w;
      }
      mbar_arrive_remote(xfree_peer);
      // valid keys of this block
      if (!warp_wait(smem_u32(&kvfull[st]), (j >> 1) & 1, TO, abort_flag)) { ok = false; break; }
      const uint64_t mask = sMask[st];
      float mblk = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        s[i] = ((mask >> i) & 1ull) ? s[i] * p.scale_log2 : -INFINITY;
        mblk = fmaxf(mblk, s[i]);
      }
      // lazy rescale: move the reference max only when it grows by more than 8 (x256)
      const bool grow = mblk > m_used + 8.0f;
      const bool need_o = grow && m_used != -INFINITY;  // O already holds earlier blocks
      if (__any_sync(0xffffffffu, need_o)) {
        if (!warp_wait(smem_u32(ofull), (j - 1) & 1, TO, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const float f = need_o ? ex2_approx(m_used - mblk) : 1.0f;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          float o[32];
          tmem_ld32(tO + c * 32 + lane_off, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= f;
          tmem_st32(tO + c * 32 + lane_off, o);
        }
        tmem_wait_st();
        l *= f;
      }
      if (grow) m_used = mblk;
      // probabilities (bf16 for the PV product; the fp32 values feed the sum)
      uint32_t pk[32];
      float lsum = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float p0 = m_used == -INFINITY ? 0.f : ex2_approx(s[2 * i] - m_used);
        const float p1 = m_used == -INFINITY ? 0.f : ex2_approx(s[2 * i + 1] - m_used);
        lsum += p0 + p1;
        pk[i] = pack_bf16x2(p0, p1);
      }
      l += lsum;
      uint8_t* pdst = sP + st * kMlaPBytes + prow;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(pdst + ((c ^ (h & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&pfull[st]));
    }
    // epilogue: O / l -> bf16, LSE
    // O is final once the last two P.V products are done; the phases are waited
    // in order because a parity wait can only tell the newest phase apart.
    if (ok && nblk > 1) ok = warp_wait(smem_u32(ofull), (nblk - 2) & 1, TO, abort_flag);
    if (ok && nblk > 0 && warp_wait(smem_u32(ofull), (nblk - 1) & 1, TO, abort_flag)) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      __nv_bfloat16* orow = p.out + (t * kMlaHeads + h) * kMlaDv + d0;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        float o[32];
        tmem_ld32(tO + c * 32 + lane_off, o);
        tmem_wait_ld();
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_uint4(pack_bf16x2(o[8 * q] * inv, o[8 * q + 1] * inv),
                              pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                              pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                              pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
      }
      if (rank == 0)
        p.lse[t * kMlaHeads + h] = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f
                                           : -INFINITY;
    }
    if (h == 0 && !seq_ok && rank == 0) report_error(kErrBounds);
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  // no CTA of the pair may leave while its peer can still touch its shared memory
  cluster_sync_all();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kMlaTmemCols);
  }
}

}  // namespace dsa
