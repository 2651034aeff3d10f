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
// [256 r, 256 r + 256) and contracts QK^T over its own 288 of the 576 key dims:
// its value dims plus half of the 64 rope dims ([512 + 32 r, 544 + 32 r)).
// Each CTA gathers its 256 value dims and the 64 rope dims of a row. The two partial
// score tiles are swapped through distributed shared memory and added
// (a + b == b + a, so both CTAs hold bit-identical scores and take identical
// softmax decisions); each CTA then runs O_r += P . V[:, its value dims].
//
// Tensor memory: O (256 columns), three score buffers of 48 columns (P, as
// bf16 pairs, later overwrites the first 24 columns of its scores) and the
// first 224 of this CTA's 288 Q dims (112 columns, two bf16 per column); the
// other 64 Q dims (the last 32 value dims and this CTA's 32 rope dims) sit in
// one 128-B-swizzled shared-memory chunk. A tcgen05.mma of M = 128, K = 16
// takes about the same time for any N up to 256, so blocks are as wide as the
// budget allows and the tensor core never waits for a free score buffer.
//
// Pipeline, per block of 48 selected keys:
//   resolver (warp 1)      turns selected indices into cache rows (-1 outside
//                          [0, pos]) and valid-key bits, four blocks at a time,
//                          for the whole row up front, into a shared table
//   gather (warps 0, 11-15) each SM's TMA unit moves only about one 128-B
//                          gathered row per ~20 cycles, and cp.async throughput
//                          grows with the number of issuing threads, so both
//                          are used side by side: warp 0 gathers rows 0-23 of
//                          the block with TMA tile::gather4 (four rows x 64
//                          dims per copy, 128-B swizzle, zero fill for row -1),
//                          warps 11-15 copy rows 24-47 in 16-B cp.async pieces
//                          (zero fill for row -1) into the same swizzled
//                          5-stage ring; both complete the stage barrier
//   MMA (warp 10)          S_j = Q . K_j^T (M=128 heads, N=48, K=288, Q from
//                          TMEM) and O += P_j . V_j (M=128, N=256, K=48, P from
//                          TMEM, V MN-major), each issued as soon as it is ready
//   softmax (warps 2-9)    thread = (head, half of the block's keys). Heads
//                          have owners: CTA r runs the online softmax of heads
//                          [64 r, 64 r + 64); its other 128 threads serve the
//                          peer's heads, sending their partial scores one block
//                          ahead and writing the P (bf16) and rescale factors
//                          the peer sends back into their TMEM lanes. Per key
//                          and direction 256 B of partial scores and 128 B of
//                          P cross the cluster (not 512 B), and each CTA
//                          exponentiates only 64 heads. Inboxes are two-buffer
//                          rings laid out [16-B chunk][head] (every warp store
//                          is 512 contiguous bytes), guarded by credits (relaxed
//                          remote mbarrier arrivals). Online softmax in base 2
//                          with a lazy rescale of O (only when the running max
//                          grows by more than 8), which the owner's factor
//                          carries to the peer's half of O.
//
// Clusters run in waves of (SMs / 2). When a call's last wave would be at most half
// full, the host may split each of its rows into key segments (consecutive parts of
// the row's selection, whole 48-key blocks) run as clusters of their own; each
// writes its segment's normalised output in fp32 and its LSE, and
// mla_combine_kernel merges them (softmax over a union of disjoint sets).
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "rows.cuh"

namespace dsa {

constexpr int kMlaHeads = 128;
constexpr int kMlaDqk = 576;
constexpr int kMlaDv = 512;
constexpr int kMlaBlk = 48;                   // keys per block
constexpr int kMlaHalf = kMlaBlk / 2;         // keys per softmax thread
constexpr int kMlaStages = 5;                 // gather ring
constexpr int kMlaSBufs = 3;                  // TMEM score / probability buffers
constexpr int kMlaXBufs = 2;                  // exchange ring (credit based)
constexpr int kMlaThreads = 512;              // TMA, resolver, 8 softmax, MMA, 5 cp.async warps
constexpr int kMlaMmaWarp = 10;
constexpr int kMlaCpWarp0 = 11;               // first cp.async warp
constexpr int kMlaCpThreads = 160;
constexpr int kMlaTmaRows = 24;               // rows of a block gathered by TMA
constexpr int kMlaKChunk = kMlaBlk * 128;     // 64-dim column chunk of a block: 6 KB
constexpr int kMlaStageBytes = 5 * kMlaKChunk;  // 4 value chunks + the 64 rope dims
constexpr int kMlaKSteps = 18;                // K = 16 steps over this CTA's 288 dims
constexpr int kMlaQCols = 112;                // TMEM columns of Q: dims [0, 224) of the slice
constexpr int kMlaQTmemSteps = kMlaQCols / 8; // K-steps whose A operand is in TMEM (14)
constexpr int kMlaQSmemBytes = kMlaHeads * 128;  // last 64 Q dims, one swizzled chunk
constexpr int kMlaMaxK = 2048;
constexpr int kMlaResolve = 4 * kMlaBlk;      // keys the resolver handles per step
constexpr int kMlaMaxSteps = (kMlaMaxK + kMlaResolve - 1) / kMlaResolve;  // 11
constexpr int kMlaRowCap = kMlaMaxSteps * kMlaResolve;                   // 2112
constexpr int kMlaMaskWords = kMlaRowCap / 32 + 2;
// Exchange inboxes, laid out [16-B chunk][64 heads of the owner] so that a
// warp's 32 heads write (and read) 512 contiguous bytes per instruction:
//   partial scores of this CTA's own heads from the peer: 12 chunks of 4 keys;
//   P (bf16) of the peer's heads from the peer: 6 chunks of 8 keys, then one
//   fp32 rescale factor per head.
constexpr int kMlaXsChunk = 64 * 16;
constexpr int kMlaXsBytes = (kMlaBlk / 4) * kMlaXsChunk;     // 12 KB
constexpr int kMlaXsPayload = kMlaXsBytes;
constexpr int kMlaXpFactor = (kMlaBlk / 8) * kMlaXsChunk;    // 6 KB of P
constexpr int kMlaXpBytes = kMlaXpFactor + 64 * 4;
constexpr int kMlaXpPayload = kMlaXpBytes;
constexpr int kMlaSmemBytes = 1024 + kMlaStages * kMlaStageBytes + kMlaQSmemBytes +
                              kMlaXBufs * (kMlaXsBytes + kMlaXpBytes) + 256 /*peer's sums*/ +
                              2 * kMlaHeads * 4 /*own sums*/ + kMlaRowCap * 4 /*rows*/ +
                              kMlaMaskWords * 4 /*valid bits*/ + 2 * 2 * kMlaHeads * 4 /*max swap*/ +
                              40 * 8 /*barriers*/ + 16;
static_assert(kMlaSmemBytes <= 232448, "sparse MLA shared memory exceeds the per-CTA limit");
constexpr uint32_t kMlaTmemCols = 512;
constexpr uint32_t kMlaTmemS = 256;           // score buffers at columns 256, 304, 352
constexpr uint32_t kMlaTmemQ = 400;           // Q: columns [400, 512)
static_assert(kMlaTmemS + kMlaSBufs * kMlaBlk <= kMlaTmemQ && kMlaTmemQ + kMlaQCols <= kMlaTmemCols,
              "sparse MLA tensor-memory plan overlaps");

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
  // Rows of a last, partly filled wave may be split into key segments: clusters
  // [0, n_whole) take whole rows (cluster c = window row c); cluster n_whole + j
  // takes segment j % nseg (keys [seg_keys (j % nseg), + seg_keys) of the row's
  // selection) of window row n_whole + j / nseg and writes that segment's
  // normalised output (fp32) and LSE to slot j of part_o / part_lse, which
  // mla_combine_kernel merges.
  int64_t n_whole;
  int32_t nseg, seg_keys;
  float* part_o;               // [slots][128][512]
  float* part_lse;             // [slots][128]
  const int32_t* q_start;      // [batch + 1] ragged query rows, or nullptr (rows.cuh)
  int32_t num_q;
};

__global__ void __launch_bounds__(kMlaThreads, 1)
    sparse_mla_kernel(const __grid_constant__ MlaParams p, const __grid_constant__ CUtensorMap tm_kv) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sKV = smem;
  uint8_t* sQ = sKV + kMlaStages * kMlaStageBytes;                      // [128][128 B] swizzled
  uint8_t* sXs = sQ + kMlaQSmemBytes;                                   // [2] partial-score inbox
  uint8_t* sXp = sXs + kMlaXBufs * kMlaXsBytes;                          // [2] P inbox
  uint8_t* sLfin = sXp + kMlaXBufs * kMlaXpBytes;                        // [64] peer's sums
  float* sLh = reinterpret_cast<float*>(sLfin + 256);                    // [2][128] own sums
  int32_t* sRow = reinterpret_cast<int32_t*>(sLh + 2 * kMlaHeads);      // [2112]
  uint32_t* sBits = reinterpret_cast<uint32_t*>(sRow + kMlaRowCap);   // valid-key bits
  float* sRed = reinterpret_cast<float*>(sBits + kMlaMaskWords);      // [2][2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRed + 2 * 2 * kMlaHeads);
  uint64_t* kvfull = bars;                     // [stages] stage landed
  uint64_t* kvempty = kvfull + kMlaStages;      // [stages] O += P V of the stage's block done
  uint64_t* sfull = kvempty + kMlaStages;       // [2] S in score buffer
  uint64_t* pfull = sfull + kMlaSBufs;          // [2] P written over S
  uint64_t* xsfull = pfull + kMlaSBufs;         // [2] peer's partial scores (own heads) arrived
  uint64_t* xsfree = xsfull + kMlaXBufs;        // [2] credit: the peer consumed our partials
  uint64_t* xpfull = xsfree + kMlaXBufs;        // [2] peer's P (its heads) arrived
  uint64_t* xpfree = xpfull + kMlaXBufs;        // [2] credit: the peer consumed our P
  uint64_t* lfull = xpfree + kMlaXBufs;         // the peer's softmax sums arrived
  uint64_t* qfull = lfull + 1;                  // Q stored in TMEM and shared memory
  uint64_t* mdone = qfull + 1;
  uint64_t* rready = mdone + 1;                 // [11] resolver step done
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(rready + kMlaMaxSteps);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int64_t cl = blockIdx.x >> 1;  // cluster
  int64_t local = cl;                  // query row within the window
  int64_t part = -1;                   // partial-output slot of a row segment
  int e0 = 0, e1 = p.k;                // this cluster's entries of the row's selection
  if (cl >= p.n_whole) {
    part = cl - p.n_whole;
    local = p.n_whole + part / p.nseg;
    e0 = (int)(part % p.nseg) * p.seg_keys;
    e1 = min(p.k, e0 + p.seg_keys);
  }
  const int b = (int)(local / p.row_count);
  const int qi = p.row_begin + (int)(local - (int64_t)b * p.row_count);
  // Position of this query row and validity of its sequence.
  const SeqRows R = seq_rows(p.q_start, p.seqlens, b, p.q_per_seq, p.num_q, p.max_ctx);
  if (qi >= R.q_len) {  // a window row the sequence does not have (ragged batch): both
    // CTAs of the pair leave before touching any barrier
    if (!R.ok && tid == 0 && rank == 0) report_error(kErrBounds);
    return;
  }
  const int64_t t = R.t0 + qi;  // global query row
  const int d0 = 256 * (int)rank;        // first value dim (and first key dim) of this CTA
  const int r0 = 512 + 32 * (int)rank;   // this CTA's quarter of the rope dims
  const bool seq_ok = R.ok;
  const int pos = R.seqlen - R.q_len + qi;
  // Blocks after the last entry inside [0, pos] hold only masked keys and change
  // nothing (no weight, no new maximum): the cluster stops at that entry's block
  // (the top-k pads a row of fewer than k visible keys with -1 at its end). Only
  // rows with fewer than k visible keys look (a uniform branch: both CTAs of the
  // pair see the same row); the others run every block.
  int nblk = (e1 - e0 + kMlaBlk - 1) / kMlaBlk;
  if (seq_ok && pos + 1 < p.k) {
    __shared__ int last_w[kMlaThreads / 32];
    int last = -1;
    for (int e = tid; e < e1 - e0; e += kMlaThreads) {
      const int sel = __ldg(p.idx + t * p.k + e0 + e);
      if (seq_ok && sel >= 0 && sel <= pos) last = e;
    }
    last = __reduce_max_sync(0xffffffffu, last);
    if (lane == 0) last_w[warp] = last;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kMlaThreads / 32; ++i) last = max(last, last_w[i]);
    nblk = max(1, (last + kMlaBlk) / kMlaBlk);  // one all-masked block when none is valid
  }

  if (tid == 0) {
    for (int i = 0; i < kMlaStages; ++i) {
      // the TMA warp's expect_tx arrival (+ its bytes) and one asynchronous
      // arrival per cp.async thread once its copies have landed
      mbar_init(smem_u32(&kvfull[i]), 1 + kMlaCpThreads);
      mbar_init(smem_u32(&kvempty[i]), 1);
    }
    for (int i = 0; i < kMlaSBufs; ++i) {
      mbar_init(smem_u32(&sfull[i]), 1);
      mbar_init(smem_u32(&pfull[i]), 256);
    }
    for (int i = 0; i < kMlaXBufs; ++i) {
      mbar_init(smem_u32(&xsfull[i]), 1);  // + the peer's bytes
      mbar_init(smem_u32(&xsfree[i]), 1);  // one remote arrival from the peer
      mbar_init(smem_u32(&xpfull[i]), 1);
      mbar_init(smem_u32(&xpfree[i]), 1);
    }
    mbar_init(smem_u32(lfull), 1);
    mbar_init(smem_u32(qfull), 256);
    mbar_init(smem_u32(mdone), 1);
    for (int i = 0; i < kMlaMaxSteps; ++i) mbar_init(smem_u32(&rready[i]), 1);
    *abort_flag = 0;
    // the first two blocks' exchange buffers start free: arm them before the
    // peer may send (later blocks are armed when their buffer is consumed)
    for (int i = 0; i < kMlaXBufs && i < nblk; ++i) {
      mbar_arrive_expect_tx(smem_u32(&xsfull[i]), kMlaXsPayload);
      mbar_arrive_expect_tx(smem_u32(&xpfull[i]), kMlaXpPayload);
    }
    mbar_arrive_expect_tx(smem_u32(lfull), 64 * 4);
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
  auto tS = [&](int j) {
    return tmem_base + kMlaTmemS + (uint32_t)kMlaBlk * (uint32_t)(j % kMlaSBufs);
  };
  const uint64_t TO = p.timeout_ns;
  int drain_dummy = 0;
  volatile int* no_abort = &drain_dummy;

  if (warp == 1) {
    // ------------------------------------------------------------ row resolver
    // Step c covers keys [192 c, 192 c + 192): lane l takes keys 192 c + 32 i + l,
    // so all six index loads (and then all six block-table loads) are in flight
    // together. No slot is ever reused, so the resolver never waits.
    const int nsteps = (nblk + 3) / 4;
    for (int c = 0; c < nsteps; ++c) {
      int sel[6], pg[6];
#pragma unroll
      for (int i = 0; i < 6; ++i) {
        const int e = c * kMlaResolve + 32 * i + lane;
        sel[i] = e0 + e < e1 ? __ldg(p.idx + t * p.k + e0 + e) : -1;
        if (!(seq_ok && sel[i] >= 0 && sel[i] <= pos)) sel[i] = -1;
      }
      if (p.paged) {
#pragma unroll
        for (int i = 0; i < 6; ++i)
          pg[i] = sel[i] >= 0 ? __ldg(p.block_table + (int64_t)b * p.max_pages + sel[i] / p.page_size)
                              : -1;
      }
#pragma unroll
      for (int i = 0; i < 6; ++i) {
        int row = -1;
        if (sel[i] >= 0) {
          if (!p.paged) {
            row = b * p.max_ctx + sel[i];
          } else if (pg[i] >= 0 && pg[i] < p.num_pages) {
            row = pg[i] * p.page_size + sel[i] % p.page_size;
          } else {
            report_error(kErrBounds);
          }
        }
        sRow[c * kMlaResolve + 32 * i + lane] = row;
        const uint32_t m = __ballot_sync(0xffffffffu, row >= 0);
        if (lane == 0) sBits[c * 6 + i] = m;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&rready[c]));  // releases the rows and bits
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA gather
    if (lane == 0) prefetch_tmap(&tm_kv);
    int issued = 0;
    for (int j = 0; j < nblk; ++j) {
      const int st = j % kMlaStages;
      // the stage is free once O += P V of block j-4 has finished
      bool ok = warp_wait(smem_u32(&kvempty[st]), ((j / kMlaStages) & 1) ^ 1, TO, abort_flag);
      if (ok && (j & 3) == 0) ok = warp_wait(smem_u32(&rready[j >> 2]), 0, TO, abort_flag);
      if (!ok) break;
      const uint32_t bar = smem_u32(&kvfull[st]);
      if (lane == 0) mbar_arrive_expect_tx(bar, kMlaTmaRows * 5 * 128);
      __syncwarp();
      if (lane < kMlaTmaRows / 4) {
        // rows 4 lane .. 4 lane + 3 of the block: value dims [d0, d0 + 256) in
        // four 64-dim chunks, then the 64 rope dims
        const int4 r = *reinterpret_cast<const int4*>(sRow + j * kMlaBlk + 4 * lane);
        const uint32_t dst = smem_u32(sKV + st * kMlaStageBytes) + lane * 4 * 128;
#pragma unroll
        for (int cb = 0; cb < 5; ++cb)
          tma_gather4(dst + cb * kMlaKChunk, &tm_kv, bar, cb < 4 ? d0 + 64 * cb : kMlaDv, r.x,
                      r.y, r.z, r.w);
      }
      issued = j + 1;
    }
    // on an early exit, let the copies still in flight land before the CTA can leave
    for (int jj = issued > kMlaStages ? issued - kMlaStages : 0; jj < issued; ++jj)
      warp_wait(smem_u32(&kvfull[jj % kMlaStages]), (jj / kMlaStages) & 1, TO, no_abort);
  } else if (warp >= kMlaCpWarp0) {
    // ------------------------------------------------------------ cp.async gather
    // rows [24, 48) of each block: 40 pieces of 16 B per row (value dims
    // [d0, d0 + 256) into chunks 0-3, the 64 rope dims into chunk 4), six per
    // thread; a warp's 32 consecutive pieces lie in one or two rows
    const int ct = tid - kMlaCpWarp0 * 32;
    for (int j = 0; j < nblk; ++j) {
      const int st = j % kMlaStages;
      bool ok = warp_wait(smem_u32(&kvempty[st]), ((j / kMlaStages) & 1) ^ 1, TO, abort_flag);
      if (ok && (j & 3) == 0) ok = warp_wait(smem_u32(&rready[j >> 2]), 0, TO, abort_flag);
      if (!ok) break;
      const uint32_t sbase = smem_u32(sKV + st * kMlaStageBytes);
#pragma unroll
      for (int i = 0; i < (kMlaBlk - kMlaTmaRows) * 40 / kMlaCpThreads; ++i) {
        const int ci = ct + i * kMlaCpThreads;
        const int kr = kMlaTmaRows + ci / 40, c = ci % 40;
        const int row = sRow[j * kMlaBlk + kr];
        const int dim = c < 32 ? d0 + 8 * c : kMlaDv + 8 * (c - 32);
        cp_async_16(sbase + (c >> 3) * kMlaKChunk + kr * 128 + (((c & 7) ^ (kr & 7)) << 4),
                    p.kv + (row >= 0 ? (int64_t)row * (kMlaDqk * 2) + dim * 2 : 0),
                    row >= 0 ? 16u : 0u);
      }
      // arrives on the stage barrier once this thread's copies have landed
      cp_async_mbar_arrive(smem_u32(&kvfull[st]));
    }
    cp_async_wait_all();
  } else if (warp == kMlaMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = instr_desc(1 /*bf16*/, 0, 0, 128, kMlaBlk);
      const uint32_t idesc_pv = instr_desc(1, 0, 1 /*V is MN-major*/, 128, 256);
      if (mbar_wait(smem_u32(qfull), 0, TO, abort_flag)) {
        tc_fence_after();
        auto issue_s = [&](int js) {  // S_js = Q . K_js^T into score buffer js % 3
          tc_fence_after();
          fence_proxy_async_smem();  // cp.async (generic proxy) writes -> tensor-core reads
          const uint32_t ka = smem_u32(sKV + (js % kMlaStages) * kMlaStageBytes);
          for (int kk = 0; kk < kMlaKSteps; ++kk) {  // 16 value + 2 rope K-steps
            // rope: this CTA's 32 dims sit at bytes [64 r, 64 r + 64) of the row
            const int kb = kk < 16 ? (kk & 3) : (kk & 3) + 2 * (int)rank;
            const uint64_t bd = smem_desc_sw128(ka + (kk >> 2) * kMlaKChunk + kb * 32, 16, 1024);
            if (kk < kMlaQTmemSteps) {
              mma_bf16_ts(tS(js), tQ + kk * 8, bd, idesc_s, kk > 0 ? 1u : 0u);
            } else {  // Q's last 64 dims: 32-B K-steps of the shared-memory chunk
              const uint64_t qd =
                  smem_desc_sw128(smem_u32(sQ) + (kk - kMlaQTmemSteps) * 32, 16, 1024);
              mma_bf16_ss(tS(js), qd, bd, idesc_s, 1u);
            }
          }
          mma_commit(smem_u32(&sfull[js % kMlaSBufs]));
        };
        auto issue_pv = [&](int jp) {  // O += P_jp . V_jp, then release the stage
          tc_fence_after();
          const uint32_t va = smem_u32(sKV + (jp % kMlaStages) * kMlaStageBytes);
#pragma unroll
          for (int kk = 0; kk < kMlaBlk / 16; ++kk) {
            const uint64_t bd = smem_desc_sw128(va + kk * 2048, kMlaKChunk, 1024);
            mma_bf16_ts(tO, tS(jp) + kk * 8, bd, idesc_pv, (jp > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(smem_u32(&kvempty[jp % kMlaStages]));
        };
        // Fixed issue order S_0, S_1, S_2, then P_j.V followed by S_{j+3} (whose
        // score buffer P_j.V frees). The softmax sends block j+1 ahead before it
        // writes P_j, so S_{j+1} is always issued before the wait for P_j. Every
        // wait suspends (try_wait), leaving issue slots to the softmax warps.
        bool go = true;
        for (int js = 0; go && js < kMlaSBufs && js < nblk; ++js) {
          go = mbar_wait(smem_u32(&kvfull[js % kMlaStages]), (js / kMlaStages) & 1, TO, abort_flag);
          if (go) issue_s(js);
        }
        for (int jp = 0; go && jp < nblk; ++jp) {
          go = mbar_wait(smem_u32(&pfull[jp % kMlaSBufs]), (jp / kMlaSBufs) & 1, TO, abort_flag);
          if (!go) break;
          issue_pv(jp);
          const int js = jp + kMlaSBufs;
          if (js < nblk) {
            go = mbar_wait(smem_u32(&kvfull[js % kMlaStages]), (js / kMlaStages) & 1, TO,
                           abort_flag);
            if (go) issue_s(js);
          }
        }
      }
      mma_commit(smem_u32(mdone));
      mbar_wait(smem_u32(mdone), 0, TO, no_abort);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    // Heads have owners: CTA r runs the online softmax of heads [64 r, 64 r + 64)
    // (its TMEM lane quadrants 2r, 2r+1). Its other 128 threads serve the peer's
    // heads: they send the peer those heads' partial scores (ahead, one block in
    // flight) and receive the peer's P (bf16) and rescale factors back into
    // their TMEM lanes. Per key and direction 256 B of partial scores and 128 B
    // of P cross the cluster instead of 512 B, and each CTA exponentiates only
    // its own 64 heads.
    const int quad = warp & 3;               // TMEM lane quadrant
    const int hf = (warp - 2) >> 2;          // which half of each block's keys
    const int h = quad * 32 + lane;          // head == TMEM lane
    const int hl = h & 63;                   // head within its owner's 64
    const int k0 = hf * kMlaHalf;            // first key (column) of this half
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool own = (h >> 6) == (int)rank;
    const bool announcer = (hf == 0 && hl == 0);  // re-arms this group's inbox, returns credits
    const uint32_t xs_off = (uint32_t)(hf * (kMlaHalf / 4)) * kMlaXsChunk + (uint32_t)hl * 16;
    const uint32_t xp_off = (uint32_t)(hf * (kMlaHalf / 8)) * kMlaXsChunk + (uint32_t)hl * 16;

    // Q slice, row h = head h. Dims [0, 224) of the slice -> TMEM lane h, two
    // bf16 per column (column c holds dims d0 + 2c, d0 + 2c + 1); this half
    // stores columns [56 hf, 56 hf + 56) in steps of 8 columns (16 dims). The
    // last 64 dims -> row h of the swizzled shared-memory chunk: half 0 stores
    // value dims [d0 + 224, d0 + 256), half 1 the rope dims [r0, r0 + 32),
    // as four 16-B pieces each.
    {
      const __nv_bfloat16* qrow = p.q + (t * kMlaHeads + h) * kMlaDqk;
      for (int c = hf * (kMlaQCols / 2); c < (hf + 1) * (kMlaQCols / 2); c += 8) {
        const uint4* src = reinterpret_cast<const uint4*>(qrow + d0 + 2 * c);
        const uint4 x0 = __ldg(src), x1 = __ldg(src + 1);
        const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        tmem_st8(tQ + c + lane_off, w);
      }
      const uint4* src = reinterpret_cast<const uint4*>(qrow + (hf == 0 ? d0 + 224 : r0));
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<uint4*>(sQ + sw128_offset((uint32_t)h, (uint32_t)(4 * hf + i))) =
            __ldg(src + i);
      fence_proxy_async_smem();  // generic-proxy stores -> tensor-core reads
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(qfull));
    }

    auto load_s = [&](int j, float* v) {  // this thread's 24 scores of block j
      tmem_ld16(tS(j) + k0 + lane_off, v);
      tmem_ld8(tS(j) + k0 + 16 + lane_off, v + 16);
      tmem_wait_ld();
    };
    // O rows of head h, this thread's 128 of the CTA's 256 value columns, x f
    auto rescale_o = [&](float f) {
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        const uint32_t col = tO + hf * 128 + c * 32 + lane_off;
        tmem_ld32(col, o);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= f;
        tmem_st32(col, o);
      }
      tmem_wait_st();
    };
    auto write_p = [&](int j, const uint32_t* pk) {  // P_j over S_j, then release it to the MMA
      tmem_st8(tS(j) + hf * (kMlaHalf / 2) + lane_off, pk);
      tmem_st4(tS(j) + hf * (kMlaHalf / 2) + 8 + lane_off, pk + 8);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&pfull[j % kMlaSBufs]));
    };

    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    if (own) {
      // ---------------------------------------------------- owner of heads h
      const uint32_t xp_peer = mapa_shared(smem_u32(sXp), peer);
      const uint32_t xpfull_peer0 = mapa_shared(smem_u32(&xpfull[0]), peer);
      const uint32_t xsfree_peer0 = mapa_shared(smem_u32(&xsfree[0]), peer);
      float cur[kMlaHalf];
      for (int j = 0; j < nblk; ++j) {
        const int xb = j % kMlaXBufs;
        float mhalf = -INFINITY;
        if (ok) ok = warp_wait(smem_u32(&sfull[j % kMlaSBufs]), (j / kMlaSBufs) & 1, TO, abort_flag);
        if (ok) {
          tc_fence_after();
          load_s(j, cur);
          ok = warp_wait<true>(smem_u32(&xsfull[xb]), (j / kMlaXBufs) & 1, TO, abort_flag);
        }
        if (ok) {  // full scores = own partial + the peer's
          const uint8_t* xr = sXs + xb * kMlaXsBytes + xs_off;
#pragma unroll
          for (int c = 0; c < kMlaHalf / 4; ++c) {
            const float4 v = *reinterpret_cast<const float4*>(xr + c * kMlaXsChunk);
            cur[4 * c] += v.x;
            cur[4 * c + 1] += v.y;
            cur[4 * c + 2] += v.z;
            cur[4 * c + 3] += v.w;
          }
          ok = warp_wait(smem_u32(&kvfull[j % kMlaStages]), (j / kMlaStages) & 1, TO, abort_flag);
        }
        if (ok) {
          const int b0 = j * kMlaBlk + k0;  // this half's 24 valid-key bits
          const uint64_t w2 = ((uint64_t)sBits[(b0 >> 5) + 1] << 32) | sBits[b0 >> 5];
          const uint32_t mask = (uint32_t)(w2 >> (b0 & 31)) & 0xFFFFFFu;
#pragma unroll
          for (int i = 0; i < kMlaHalf; ++i) {
            cur[i] = ((mask >> i) & 1u) ? cur[i] * p.scale_log2 : -INFINITY;
            mhalf = fmaxf(mhalf, cur[i]);
          }
          sRed[((j & 1) * 2 + hf) * kMlaHeads + h] = mhalf;
        }
        // both halves of a head agree on the block max (and on whether to go on)
        tc_fence_before();
        if (!named_barrier_and(2, 128, ok)) break;
        tc_fence_after();
        // every owner thread has read inbox xb: re-arm it for block j+2 and hand
        // the peer the credit (relaxed: the values are consumed)
        if (announcer && j + kMlaXBufs < nblk) {
          mbar_arrive_expect_tx(smem_u32(&xsfull[xb]), kMlaXsPayload);
          mbar_arrive_remote_relaxed(xsfree_peer0 + (uint32_t)xb * 8u);
        }
        const float mblk =
            fmaxf(sRed[((j & 1) * 2) * kMlaHeads + h], sRed[((j & 1) * 2 + 1) * kMlaHeads + h]);
        // lazy rescale: move the reference max only when it grows by more than 8 (x256)
        const bool grow = mblk > m_used + 8.0f;
        const bool need_o = grow && m_used != -INFINITY;  // O already holds earlier blocks
        const float f = need_o ? ex2_approx(m_used - mblk) : 1.0f;
        if (__any_sync(0xffffffffu, need_o)) {
          // O += P_{j-1} V_{j-1} must have finished before O is touched
          if (!warp_wait(smem_u32(&kvempty[(j - 1) % kMlaStages]), ((j - 1) / kMlaStages) & 1, TO,
                         abort_flag)) {
            ok = false;
          } else {
            tc_fence_after();
            rescale_o(f);
          }
        }
        l *= f;
        if (grow) m_used = mblk;
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
        // P_j and the factor to the peer (its inbox xb is free once it has
        // consumed block j-2 and returned the credit)
        if (ok && j >= kMlaXBufs)
          ok = warp_wait<true>(smem_u32(&xpfree[xb]), ((j / kMlaXBufs) - 1) & 1, TO, abort_flag);
        if (ok) {
          const uint32_t dst = xp_peer + xb * kMlaXpBytes + xp_off;
          const uint32_t bar = xpfull_peer0 + xb * 8;
#pragma unroll
          for (int c = 0; c < kMlaHalf / 8; ++c)
            st_async_v4u(dst + c * kMlaXsChunk, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                         pk[4 * c + 3], bar);
          if (hf == 0)
            st_async_u32(xp_peer + xb * kMlaXpBytes + kMlaXpFactor + hl * 4, __float_as_uint(f),
                         bar);
        }
        write_p(j, pk);
      }
    } else {
      // ---------------------------------------------------- server of the peer's heads h
      const uint32_t xs_peer = mapa_shared(smem_u32(sXs), peer);
      const uint32_t xsfull_peer0 = mapa_shared(smem_u32(&xsfull[0]), peer);
      const uint32_t xpfree_peer0 = mapa_shared(smem_u32(&xpfree[0]), peer);
      // Block j's partial scores of these heads, from TMEM to the owner's inbox
      // j % 2 (free from block 2 on once the owner consumed block j-2).
      auto load_and_send = [&](int j) {
        float v[kMlaHalf];
        bool r = warp_wait(smem_u32(&sfull[j % kMlaSBufs]), (j / kMlaSBufs) & 1, TO, abort_flag);
        if (r && j >= kMlaXBufs)
          r = warp_wait<true>(smem_u32(&xsfree[j % kMlaXBufs]), ((j / kMlaXBufs) - 1) & 1, TO,
                              abort_flag);
        if (r) {
          tc_fence_after();
          load_s(j, v);
          const uint32_t xb = (uint32_t)(j % kMlaXBufs);
          const uint32_t dst = xs_peer + xb * kMlaXsBytes + xs_off;
          const uint32_t bar = xsfull_peer0 + xb * 8;
#pragma unroll
          for (int c = 0; c < kMlaHalf / 4; ++c)
            st_async_v4(dst + c * kMlaXsChunk, v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3],
                        bar);
        }
        return r;
      };
      if (nblk > 0) ok = load_and_send(0);
      for (int j = 0; j < nblk; ++j) {
        const int xb = j % kMlaXBufs;
        // send ahead: block j+1 leaves before block j's P is awaited
        if (ok && j + 1 < nblk) ok = load_and_send(j + 1);
        uint32_t pk[kMlaHalf / 2];
        float f = 1.0f;
        if (ok) ok = warp_wait<true>(smem_u32(&xpfull[xb]), (j / kMlaXBufs) & 1, TO, abort_flag);
        if (ok) {
          const uint8_t* xr = sXp + xb * kMlaXpBytes + xp_off;
#pragma unroll
          for (int c = 0; c < kMlaHalf / 8; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(xr + c * kMlaXsChunk);
            pk[4 * c] = v.x;
            pk[4 * c + 1] = v.y;
            pk[4 * c + 2] = v.z;
            pk[4 * c + 3] = v.w;
          }
          f = *reinterpret_cast<const float*>(sXp + xb * kMlaXpBytes + kMlaXpFactor + hl * 4);
        } else {
#pragma unroll
          for (int i = 0; i < kMlaHalf / 2; ++i) pk[i] = 0u;
        }
        tc_fence_before();
        if (!named_barrier_and(3, 128, ok)) break;
        tc_fence_after();
        if (announcer && j + kMlaXBufs < nblk) {
          mbar_arrive_expect_tx(smem_u32(&xpfull[xb]), kMlaXpPayload);
          mbar_arrive_remote_relaxed(xpfree_peer0 + (uint32_t)xb * 8u);
        }
        // the owner moved its reference max: rescale these heads' O rows too
        if (__any_sync(0xffffffffu, f != 1.0f)) {
          if (!warp_wait(smem_u32(&kvempty[(j - 1) % kMlaStages]), ((j - 1) / kMlaStages) & 1, TO,
                         abort_flag)) {
            ok = false;
          } else {
            tc_fence_after();
            rescale_o(f);
          }
        }
        write_p(j, pk);
      }
    }

    // ------------------------------------------------------------------ epilogue
    // every P.V product has finished once the last one has (in order)
    if (ok && nblk > 0)
      ok = warp_wait(smem_u32(&kvempty[(nblk - 1) % kMlaStages]), ((nblk - 1) / kMlaStages) & 1,
                     TO, abort_flag);
    if (own) sLh[hf * kMlaHeads + h] = l;
    tc_fence_before();
    const bool all_ok = named_barrier_and(4, 256, ok);
    tc_fence_after();
    float lt = 0.f;
    bool lt_ok = all_ok;
    if (own) {
      lt = sLh[h] + sLh[kMlaHeads + h];
      if (hf == 0) {
        // the peer normalises its half of these heads' rows with the same sum
        st_async_u32(mapa_shared(smem_u32(sLfin), peer) + hl * 4, __float_as_uint(lt),
                     mapa_shared(smem_u32(lfull), peer));
        if (all_ok) {
          const float lse_h =
              lt > 0.f ? (m_used + __log2f(lt)) * 0.69314718055994531f : -INFINITY;
          if (part < 0) {
            p.lse[t * kMlaHeads + h] = lse_h;
          } else {
            p.part_lse[part * kMlaHeads + h] = lse_h;
          }
        }
      }
    } else {
      lt_ok = warp_wait<true>(smem_u32(lfull), 0, TO, abort_flag) && all_ok;
      if (lt_ok) lt = reinterpret_cast<const float*>(sLfin)[hl];
    }
    if (lt_ok && nblk > 0 && part >= 0) {  // a row segment: fp32 for the merge
      const float inv = lt > 0.f ? 1.0f / lt : 0.f;
      float* prow = p.part_o + (part * kMlaHeads + h) * kMlaDv + d0 + hf * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(tO + hf * 128 + c * 32 + lane_off, o);
        tmem_wait_ld();
        float4* dst = reinterpret_cast<float4*>(prow + c * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = make_float4(o[4 * q] * inv, o[4 * q + 1] * inv, o[4 * q + 2] * inv,
                               o[4 * q + 3] * inv);
      }
    } else if (lt_ok && nblk > 0) {
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

// Merge of a row's key segments (the same attention, split over disjoint parts of
// S_t): with segment LSEs l_s and normalised outputs o_s,
//   LSE = ln sum_s e^{l_s},   o = sum_s e^{l_s - LSE} o_s,
// and LSE = -inf, o = 0 when no segment holds a valid key (as for a whole row).
constexpr int kMlaMaxSeg = 8;
struct MlaCombineParams {
  const float* part_o;  // [slots][128][512]
  const float* part_lse;  // [slots][128]
  __nv_bfloat16* out;
  float* lse;
  int64_t n_whole;
  int32_t nseg, row_begin, row_count, q_per_seq;
  const int32_t* q_start;  // [batch + 1] ragged query rows, or nullptr (rows.cuh)
  const int32_t* seqlens;
  int32_t num_q, max_ctx;
};

// grid (split rows, 16), 256 threads: warp = one of 8 heads, lane = 16 value dims
__global__ void __launch_bounds__(256) mla_combine_kernel(const __grid_constant__ MlaCombineParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t j = blockIdx.x;
  const int h = blockIdx.y * 8 + warp;
  const int64_t local = p.n_whole + j;
  const int b = (int)(local / p.row_count);
  const int qi = p.row_begin + (int)(local - (int64_t)b * p.row_count);
  const SeqRows R = seq_rows(p.q_start, p.seqlens, b, p.q_per_seq, p.num_q, p.max_ctx);
  if (qi >= R.q_len) return;  // no such row: its segments never ran
  const int64_t t = R.t0 + qi;
  float l[kMlaMaxSeg];
  float m = -INFINITY;
#pragma unroll
  for (int s = 0; s < kMlaMaxSeg; ++s) {
    l[s] = s < p.nseg ? __ldg(p.part_lse + (j * p.nseg + s) * kMlaHeads + h) : -INFINITY;
    m = fmaxf(m, l[s]);
  }
  float o[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i] = 0.f;
  float lse_t = -INFINITY;
  if (m != -INFINITY) {
    float sum = 0.f;
#pragma unroll
    for (int s = 0; s < kMlaMaxSeg; ++s) sum += s < p.nseg ? expf(l[s] - m) : 0.f;
    lse_t = m + logf(sum);
#pragma unroll
    for (int s = 0; s < kMlaMaxSeg; ++s) {
      const float a = s < p.nseg ? expf(l[s] - lse_t) : 0.f;
      if (a == 0.f) continue;  // warp-uniform: past nseg, or an empty or negligible segment
      const float4* src = reinterpret_cast<const float4*>(
          p.part_o + ((j * p.nseg + s) * kMlaHeads + h) * kMlaDv + lane * 16);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = __ldg(src + q);
        o[4 * q] = fmaf(a, v.x, o[4 * q]);
        o[4 * q + 1] = fmaf(a, v.y, o[4 * q + 1]);
        o[4 * q + 2] = fmaf(a, v.z, o[4 * q + 2]);
        o[4 * q + 3] = fmaf(a, v.w, o[4 * q + 3]);
      }
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(p.out + (t * kMlaHeads + h) * kMlaDv + lane * 16);
  dst[0] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                      pack_bf16x2(o[6], o[7]));
  dst[1] = make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]),
                      pack_bf16x2(o[12], o[13]), pack_bf16x2(o[14], o[15]));
  if (lane == 0) p.lse[t * kMlaHeads + h] = lse_t;
}

}  // namespace dsa
