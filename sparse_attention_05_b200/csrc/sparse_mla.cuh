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
// score tiles are swapped through distributed shared memory and added
// (a + b == b + a, so both CTAs hold bit-identical scores and take identical
// softmax decisions); each CTA then runs O_r += P . V[:, its value dims].
//
// Tensor memory: O (256 columns), three score buffers of 32 columns (P, as
// bf16 pairs, later overwrites the first 16 columns of its scores) and this
// CTA's slice of Q (128 or 160 columns, two bf16 per column): Q and P are read
// by the tensor core straight from tensor memory, which leaves shared memory to
// a deep gather ring and the exchange buffers.
//
// Pipeline, per block of 32 selected keys:
//   producers (warps 0-1)  resolve cache rows one block ahead and gather the
//                          rows' slice with cp.async (zero fill for entries
//                          outside [0, pos]) into a 6-stage 128-B-swizzled ring;
//                          completion arrives asynchronously on the stage barrier
//   MMA (warp 10)          S_j = Q . K_j^T (M=128 heads, N=32, K=256|320, Q from
//                          TMEM) and O += P_j . V_j (M=128, N=256, K=32, P from
//                          TMEM, V MN-major), each issued as soon as it is ready
//   softmax (warps 2-9)    thread = (head, half of the block's keys). Block j+1's
//                          partial scores go to the peer before block j's softmax
//                          runs; four exchange buffers mean the peer can only
//                          overwrite a buffer after a chain of data dependencies
//                          through this CTA's later sends, so no handshake is
//                          needed. Online softmax in base 2 with a lazy rescale
//                          of O (only when the running max grows by more than 8).
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dsa {

constexpr int kMlaHeads = 128;
constexpr int kMlaDqk = 576;
constexpr int kMlaDv = 512;
constexpr int kMlaBlk = 32;                   // keys per block
constexpr int kMlaHalf = kMlaBlk / 2;         // keys per softmax thread
constexpr int kMlaStages = 6;                 // gather ring
constexpr int kMlaSBufs = 3;                  // TMEM score / probability buffers
constexpr int kMlaXBufs = 4;                  // exchange buffers
constexpr int kMlaThreads = 352;              // 2 producer, 8 softmax, 1 MMA warp
constexpr int kMlaMmaWarp = 10;
constexpr int kMlaKChunk = kMlaBlk * 128;     // 64-dim column chunk of a block: 4 KB
constexpr int kMlaStageBytes = 5 * kMlaKChunk;
constexpr int kMlaXRow = 36;                  // floats per exchange row (32 + pad)
constexpr int kMlaXBytes = kMlaHeads * kMlaXRow * 4;
constexpr int kMlaXPayload = kMlaHeads * kMlaBlk * 4;  // bytes the peer sends per block
constexpr int kMlaSmemBytes = 1024 + kMlaStages * kMlaStageBytes + kMlaXBufs * kMlaXBytes +
                              kMlaStages * kMlaBlk * 4 /*rows*/ + 8 * 4 /*masks*/ +
                              2 * 2 * kMlaHeads * 4 /*max swap*/ + 32 * 8 /*barriers*/ + 16;
constexpr uint32_t kMlaTmemCols = 512;
constexpr uint32_t kMlaTmemS = 256;           // score buffers at 256, 288, 320
constexpr uint32_t kMlaTmemQ = 352;           // Q slice: 128 or 160 columns

struct MlaParams {
  const uint8_t* kv;           // latent cache rows of 1152 B
  const __nv_bfloat16* q;      // [T][128][576]
  const int32_t* idx;          // [T][k]
  const int32_t* block_table;  // paged
  const int32_t* seqlens;      // [batch] or nullptr
  __nv_bfloat16* out;          // [T][128][512]
  float* lse;                  // [T][128]
  int32_t k, batch, max_ctx, q_per_seq;
  int32_t row_begin, row_count;  // window of rows per sequence
  int32_t paged, page_size, max_pages, num_pages;
  int64_t cache_rows;
  float scale_log2;            // scale * log2(e)
  uint64_t timeout_ns;
};

__global__ void __launch_bounds__(kMlaThreads, 1) sparse_mla_kernel(const __grid_constant__ MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sKV = smem;
  uint8_t* sX = sKV + kMlaStages * kMlaStageBytes;                      // [4][128][36] f32
  int32_t* sRow = reinterpret_cast<int32_t*>(sX + kMlaXBufs * kMlaXBytes);   // [6][32]
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sRow + kMlaStages * kMlaBlk);  // [8]
  float* sRed = reinterpret_cast<float*>(sMask + 8);                  // [2][2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRed + 2 * 2 * kMlaHeads);
  uint64_t* kvfull = bars + 0;     // [6] stage landed + mask published
  uint64_t* kvempty = bars + 6;    // [6] O += P V of the stage's block done
  uint64_t* sfull = bars + 12;     // [3] S in score buffer
  uint64_t* pfull = bars + 15;     // [3] P written over S
  uint64_t* xfull = bars + 18;     // [4] peer's partial scores arrived
  uint64_t* qfull = bars + 22;     // Q stored in TMEM
  uint64_t* mdone = bars + 23;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int64_t local = blockIdx.x >> 1;  // query row within the window
  const int b = (int)(local / p.row_count);
  const int qi = p.row_begin + (int)(local - (int64_t)b * p.row_count);
  const int64_t t = (int64_t)b * p.q_per_seq + qi;  // global query row
  const int nchunk = 4 + (int)rank;      // 64-dim column chunks of this CTA's key slice
  const int d0 = 256 * (int)rank;        // first key dim of the slice (also first value dim)
  const int nblk = (p.k + kMlaBlk - 1) / kMlaBlk;

  if (tid == 0) {
    for (int i = 0; i < kMlaStages; ++i) {
      mbar_init(smem_u32(&kvfull[i]), 64 + 1);  // 64 async cp.async arrivals + mask writer
      mbar_init(smem_u32(&kvempty[i]), 1);
    }
    for (int i = 0; i < kMlaSBufs; ++i) {
      mbar_init(smem_u32(&sfull[i]), 1);
      mbar_init(smem_u32(&pfull[i]), 256);
    }
    for (int i = 0; i < kMlaXBufs; ++i) mbar_init(smem_u32(&xfull[i]), 1);  // + peer's bytes
    mbar_init(smem_u32(qfull), 256);
    mbar_init(smem_u32(mdone), 1);
    *abort_flag = 0;
    fence_mbarrier_init_cluster();
  }
  if (warp == kMlaMmaWarp) {
    tmem_alloc(smem_u32(tmem_holder), kMlaTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  // Both CTAs' barriers must be initialised before the peer may touch them.
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t tO = tmem_base;
  const uint32_t tQ = tmem_base + kMlaTmemQ;
  auto tS = [&](int j) { return tmem_base + kMlaTmemS + 32u * (uint32_t)(j % kMlaSBufs); };
  const uint64_t TO = p.timeout_ns;
  int drain_dummy = 0;
  volatile int* no_abort = &drain_dummy;

  // Position of this query row and validity of its sequence.
  const int seqlen = p.seqlens ? __ldg(p.seqlens + b) : p.max_ctx;
  const bool seq_ok = seqlen >= p.q_per_seq && seqlen <= p.max_ctx;
  const int pos = seqlen - p.q_per_seq + qi;

  if (warp < 2) {
    // ------------------------------------------------------------ gather producers
    const int nch16 = nchunk * 8;  // 16-byte chunks per row slice
    // Cache rows of block j into sRow[j % 6] (-1: outside [0, pos], zero-filled)
    // and its valid-key mask into sMask[j & 7].
    auto rows_for = [&](int j) {
      if (warp == 0) {
        const int e = j * kMlaBlk + lane;
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
        sRow[(j % kMlaStages) * kMlaBlk + lane] = row;
        const uint32_t m = __ballot_sync(0xffffffffu, row >= 0);
        if (lane == 0) sMask[j & 7] = m;
      }
    };
    if (nblk > 0) rows_for(0);
    for (int j = 0; j < nblk; ++j) {
      const int st = j % kMlaStages;
      // The stage is free once O += P V of block j-6 has finished. Both producer
      // warps decide together (neither is left behind in a barrier when a wait
      // gives up); the barrier also publishes sRow[st].
      const bool ok = warp_wait(smem_u32(&kvempty[st]), ((j / kMlaStages) & 1) ^ 1, TO, abort_flag);
      if (!named_barrier_and(1, 64, ok)) break;
      {
        // two threads per key row: chunks c = (tid & 1), (tid & 1) + 2, ...
        const int kr = tid >> 1;
        const int row = sRow[st * kMlaBlk + kr];
        const uint8_t* src = p.kv + (row >= 0 ? (int64_t)row * (kMlaDqk * 2) : 0) + d0 * 2;
        const uint32_t dst = smem_u32(sKV + st * kMlaStageBytes) + kr * 128;
        const uint32_t nbytes = row >= 0 ? 16u : 0u;
        for (int c = tid & 1; c < nch16; c += 2)
          cp_async_16(dst + (c >> 3) * kMlaKChunk + (((c & 7) ^ (kr & 7)) << 4), src + c * 16,
                      nbytes);
      }
      // this thread's copies arrive on kvfull[st] when they land (no waiting here)
      cp_async_mbar_arrive(smem_u32(&kvfull[st]));
      // the block's mask word (written one block earlier) is released by its writer
      if (tid == 0) mbar_arrive(smem_u32(&kvfull[st]));
      if (j + 1 < nblk) rows_for(j + 1);
    }
    cp_async_wait_all();
    __syncwarp();
  } else if (warp == kMlaMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = instr_desc(1 /*bf16*/, 0, 0, 128, kMlaBlk);
      const uint32_t idesc_pv = instr_desc(1, 0, 1 /*V is MN-major*/, 128, 256);
      if (mbar_wait(smem_u32(qfull), 0, TO, abort_flag)) {
        tc_fence_after();
        // Issue S_j (needs block j landed and P_{j-3}.V issued: its score buffer
        // is reused) and P_i.V (needs P_i written) in order of readiness; the
        // barriers are tested without suspending, so neither waits on the other.
        int js = 0, jp = 0;
        uint64_t t_last = globaltimer_ns();
        uint32_t spins = 0;
        while (jp < nblk && !*abort_flag) {
          bool progressed = false;
          if (js < nblk && js < jp + kMlaSBufs &&
              mbar_test_wait(smem_u32(&kvfull[js % kMlaStages]), (js / kMlaStages) & 1)) {
            fence_proxy_async_smem();  // cp.async writes -> tensor-core reads
            tc_fence_after();
            const uint32_t ka = smem_u32(sKV + (js % kMlaStages) * kMlaStageBytes);
            for (int kk = 0; kk < nchunk * 4; ++kk) {
              const uint64_t bd =
                  smem_desc_sw128(ka + (kk >> 2) * kMlaKChunk + (kk & 3) * 32, 16, 1024);
              mma_bf16_ts(tS(js), tQ + kk * 8, bd, idesc_s, kk > 0 ? 1u : 0u);
            }
            mma_commit(smem_u32(&sfull[js % kMlaSBufs]));
            ++js;
            progressed = true;
          }
          if (jp < js && mbar_test_wait(smem_u32(&pfull[jp % kMlaSBufs]), (jp / kMlaSBufs) & 1)) {
            tc_fence_after();
            const uint32_t va = smem_u32(sKV + (jp % kMlaStages) * kMlaStageBytes);
#pragma unroll
            for (int kk = 0; kk < kMlaBlk / 16; ++kk) {
              const uint64_t bd = smem_desc_sw128(va + kk * 2048, kMlaKChunk, 1024);
              mma_bf16_ts(tO, tS(jp) + kk * 8, bd, idesc_pv, (jp > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(smem_u32(&kvempty[jp % kMlaStages]));
            ++jp;
            progressed = true;
          }
          if (progressed) {
            t_last = globaltimer_ns();
          } else if ((++spins & 63) == 0 && globaltimer_ns() - t_last > TO) {
            report_error(kErrTimeout);  // neither input became ready in time
            *abort_flag = 1;
          }
        }
      }
      mma_commit(smem_u32(mdone));
      mbar_wait(smem_u32(mdone), 0, TO, no_abort);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int quad = warp & 3;               // TMEM lane quadrant
    const int hf = (warp - 2) >> 2;          // which half of each block's keys
    const int h = quad * 32 + lane;          // head == TMEM lane
    const int k0 = hf * kMlaHalf;            // first key (column) of this half
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t x_peer = mapa_shared(smem_u32(sX), peer);
    const uint32_t xfull_peer0 = mapa_shared(smem_u32(&xfull[0]), peer);
    const uint32_t xrow_off = (uint32_t)h * (kMlaXRow * 4) + (uint32_t)k0 * 4;
    const bool announcer = (hf == 0 && h == 0);  // arms this CTA's xfull phases

    // Q slice -> TMEM (row h = lane h): this half stores columns
    // [hf * qcols/2, (hf + 1) * qcols/2), two bf16 per column.
    {
      const int qcols = 32 * nchunk;
      const int c0 = hf * (qcols / 2);
      const uint4* src = reinterpret_cast<const uint4*>(
          p.q + (t * kMlaHeads + h) * kMlaDqk + d0 + 2 * c0);
      for (int c = 0; c < qcols / 2; c += 16) {  // 16 columns = 32 dims = 64 B per step
        uint32_t w[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 x = __ldg(src + (c / 4) + v);
          w[4 * v] = x.x;
          w[4 * v + 1] = x.y;
          w[4 * v + 2] = x.z;
          w[4 * v + 3] = x.w;
        }
        tmem_st8(tQ + c0 + c + lane_off, w);
        tmem_st8(tQ + c0 + c + 8 + lane_off, w + 8);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(qfull));
    }

    auto load_s = [&](int j, float* v) {  // this thread's 16 scores of block j
      tmem_ld16(tS(j) + k0 + lane_off, v);
      tmem_wait_ld();
    };
    auto send = [&](int j, const float* v) {  // partial scores of block j -> peer
      const uint32_t xb = (uint32_t)(j & (kMlaXBufs - 1));
      const uint32_t dst = x_peer + xb * kMlaXBytes + xrow_off;
      const uint32_t bar = xfull_peer0 + xb * 8;
#pragma unroll
      for (int c = 0; c < kMlaHalf / 4; ++c)
        st_async_v4(dst + c * 16, v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3], bar);
    };

    float m_used = -INFINITY, l = 0.f;
    float cur[kMlaHalf], nxt[kMlaHalf];
#pragma unroll
    for (int i = 0; i < kMlaHalf; ++i) cur[i] = nxt[i] = 0.f;
    bool ok = true;
    // prologue: block 0's partial goes out first
    if (nblk > 0) {
      if (announcer) mbar_arrive_expect_tx(smem_u32(&xfull[0]), kMlaXPayload);
      ok = warp_wait(smem_u32(&sfull[0]), 0, TO, abort_flag);
      if (ok) {
        tc_fence_after();
        load_s(0, cur);
        send(0, cur);
      }
    }
    for (int j = 0; j < nblk; ++j) {
      const int xb = j & (kMlaXBufs - 1);
      // (A) block j+1: scores from TMEM, partial sent to the peer. Its buffer
      // was last used for block j-3, which this CTA consumed three blocks ago,
      // before sending blocks j-1 and j that the peer has waited on since.
      if (ok && j + 1 < nblk) {
        if (announcer)
          mbar_arrive_expect_tx(smem_u32(&xfull[(j + 1) & (kMlaXBufs - 1)]), kMlaXPayload);
        ok = warp_wait(smem_u32(&sfull[(j + 1) % kMlaSBufs]), ((j + 1) / kMlaSBufs) & 1, TO,
                       abort_flag);
        if (ok) {
          tc_fence_after();
          load_s(j + 1, nxt);
          send(j + 1, nxt);
        }
      }
      // (B) block j: full scores = own partial + the peer's
      float mhalf = -INFINITY;
      if (ok) ok = warp_wait<true>(smem_u32(&xfull[xb]), (j >> 2) & 1, TO, abort_flag);
      if (ok) {
        const float* xr = reinterpret_cast<const float*>(sX + xb * kMlaXBytes + xrow_off);
#pragma unroll
        for (int c = 0; c < kMlaHalf / 4; ++c) {
          const float4 v = reinterpret_cast<const float4*>(xr)[c];
          cur[4 * c] += v.x;
          cur[4 * c + 1] += v.y;
          cur[4 * c + 2] += v.z;
          cur[4 * c + 3] += v.w;
        }
        ok = warp_wait(smem_u32(&kvfull[j % kMlaStages]), (j / kMlaStages) & 1, TO, abort_flag);
      }
      if (ok) {
        const uint32_t mask = (sMask[j & 7] >> k0) & 0xFFFFu;
#pragma unroll
        for (int i = 0; i < kMlaHalf; ++i) {
          cur[i] = ((mask >> i) & 1u) ? cur[i] * p.scale_log2 : -INFINITY;
          mhalf = fmaxf(mhalf, cur[i]);
        }
        sRed[((j & 1) * 2 + hf) * kMlaHeads + h] = mhalf;
      }
      // both halves of a head agree on the block max (and on whether to go on)
      tc_fence_before();
      if (!named_barrier_and(2, 256, ok)) break;
      tc_fence_after();
      const float mblk =
          fmaxf(sRed[((j & 1) * 2) * kMlaHeads + h], sRed[((j & 1) * 2 + 1) * kMlaHeads + h]);
      // lazy rescale: move the reference max only when it grows by more than 8 (x256)
      const bool grow = mblk > m_used + 8.0f;
      const bool need_o = grow && m_used != -INFINITY;  // O already holds earlier blocks
      if (__any_sync(0xffffffffu, need_o)) {
        // O += P_{j-1} V_{j-1} must have finished before O is touched
        if (!warp_wait(smem_u32(&kvempty[(j - 1) % kMlaStages]), ((j - 1) / kMlaStages) & 1, TO,
                       abort_flag)) {
          ok = false;
        } else {
          tc_fence_after();
          const float f = need_o ? ex2_approx(m_used - mblk) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {  // this half's 128 columns of O
            float o[32];
            const uint32_t col = tO + hf * 128 + c * 32 + lane_off;
            tmem_ld32(col, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= f;
            tmem_st32(col, o);
          }
          tmem_wait_st();
          l *= f;
        }
      }
      if (grow) m_used = mblk;
      if (ok) {
        // probabilities: bf16 for the PV product, fp32 for the normaliser
        uint32_t pk[kMlaHalf / 2];
        float lsum = 0.f;
#pragma unroll
        for (int i = 0; i < kMlaHalf / 2; ++i) {
          const float p0 = m_used == -INFINITY ? 0.f : ex2_approx(cur[2 * i] - m_used);
          const float p1 = m_used == -INFINITY ? 0.f : ex2_approx(cur[2 * i + 1] - m_used);
          lsum += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        l += lsum;
        // P_j over S_j: packed columns [8 hf, 8 hf + 8) of score buffer j
        tmem_st8(tS(j) + hf * (kMlaHalf / 2) + lane_off, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&pfull[j % kMlaSBufs]));
      }
#pragma unroll
      for (int i = 0; i < kMlaHalf; ++i) cur[i] = nxt[i];
    }
    // epilogue: every P.V product has finished once the last one has (in order)
    if (ok && nblk > 0)
      ok = warp_wait(smem_u32(&kvempty[(nblk - 1) % kMlaStages]), ((nblk - 1) / kMlaStages) & 1,
                     TO, abort_flag);
    // the two halves' normalisers meet in exchange buffer 0: nothing arrives
    // there any more (the peer's last block has been consumed), while the max
    // swap slots may still be read by the other half of this head
    float* sL = reinterpret_cast<float*>(sX);
    sL[hf * kMlaHeads + h] = l;
    tc_fence_before();
    const bool all_ok = named_barrier_and(2, 256, ok);
    tc_fence_after();
    if (all_ok && nblk > 0) {
      const float lt = sL[h] + sL[kMlaHeads + h];
      const float inv = lt > 0.f ? 1.0f / lt : 0.f;
      __nv_bfloat16* orow = p.out + (t * kMlaHeads + h) * kMlaDv + d0 + hf * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(tO + hf * 128 + c * 32 + lane_off, o);
        tmem_wait_ld();
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_uint4(pack_bf16x2(o[8 * q] * inv, o[8 * q + 1] * inv),
                              pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                              pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                              pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
      }
      if (rank == 0 && hf == 0)
        p.lse[t * kMlaHeads + h] = lt > 0.f ? (m_used + __log2f(lt)) * 0.69314718055994531f
                                            : -INFINITY;
    }
    if (h == 0 && hf == 0 && !seq_ok && rank == 0) report_error(kErrBounds);
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  // no CTA of the pair may leave while its peer can still touch its shared memory
  cluster_sync_all();
  if (warp == kMlaMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kMlaTmemCols);
  }
}

}  // namespace dsa
