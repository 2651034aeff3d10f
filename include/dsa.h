/*
 * dsa.h -- C ABI of the B200 (sm_100a) DeepSeek Sparse Attention forward.
 *
 * The forward of DSA as the DeepSeek-V3.2-Exp technical report defines it
 * (Chinese translation on m.163.com, §1 "Architecture"):
 *   1. lightning indexer  I_{t,s} = sum_j w_{t,j} * ReLU(q^I_{t,j} . k^I_s)   (Eq. 1)
 *      over the H^I = 64 indexer heads, keys s <= pos(t) (causal);
 *   2. fine-grained token selection S_t = Top-k(I_{t,:}), k <= 2048        (§1, §2.1)
 *   3. sparse MLA in MQA mode: every one of the 128 query heads attends over
 *      the selected shared latent rows c_s (576-d key = 512 latent + 64 rope,
 *      value = first 512 dims), u_t = Attn(h_t, {c_s : s in S_t})           (Eq. 2, Fig. 1)
 * The 128-d FP8 indexer key cache and the 512-d latent cache are the two
 * per-token caches of "DeepSeek-V3.2开源技术报告" (nsmao.com, DSA principle).
 *
 * Conventions shared by every entry point
 *  - All tensor arguments are device pointers to caller-owned memory,
 *    row-major and dense, 16-byte aligned. The library allocates no memory.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream). Host-side argument checks return an error status
 *    synchronously and launch nothing. Conditions only the device can see
 *    (a sequence shorter than its query rows, a block-table entry outside the
 *    cache, a bounded wait that ran out) set a device error word, read and
 *    cleared by dsa_get_device_error(); the affected outputs are unspecified.
 *  - The kernels are compiled for fixed dimensions: H^I = 64, d_I = 128,
 *    H = 128 query heads, D = 576, D_v = 512, 1 <= k <= 2048, page size a
 *    multiple of 64. Anything else returns DSA_ERR_UNSUPPORTED_SHAPE; there is
 *    no fallback path.
 *  - Query geometry: the query rows of sequence b are its last q_len[b] tokens
 *    (decode: the 1 or 2 newest; prefill: the whole prompt; chunked prefill: the
 *    chunk just appended to a cache that already holds the earlier tokens). Row i
 *    of sequence b (0 <= i < q_len[b]) is global query row t = t0[b] + i at
 *    position pos(t) = seqlen[b] - q_len[b] + i, and sees keys s in [0, pos(t)].
 *    Uniform batch (dsa_q_desc_t.q_start == NULL): q_len[b] = q_per_seq and
 *    t0[b] = b * q_per_seq. Ragged batch: t0[b] = q_start[b] and
 *    q_len[b] = q_start[b + 1] - q_start[b] (see dsa_q_desc_t).
 *  - Thread safety: calls may be issued from several host threads; calls
 *    that overlap on the GPU share only the device error word.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

/* Same object as cudaStream_t; declared here so callers need no CUDA header. */
typedef struct CUstream_st* dsa_stream_t;

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,       /* null pointer, bad size or alignment          */
  DSA_ERR_UNSUPPORTED_SHAPE = 2, /* dims other than the compiled ones             */
  DSA_ERR_CUDA = 3,              /* a CUDA runtime call failed                    */
  DSA_ERR_DEVICE_TIMEOUT = 4,    /* a bounded device-side wait ran out            */
  DSA_ERR_BOUNDS = 5,            /* device saw an index / page / length out of range */
  DSA_ERR_WORKSPACE = 6          /* workspace missing or smaller than required    */
} dsa_status_t;

typedef enum { DSA_KV_CONTIGUOUS = 0, DSA_KV_PAGED = 1 } dsa_kv_layout_t;

/* Geometry of the two per-token caches (indexer keys and MLA latents share it).
 *  contiguous: token s of sequence b is row b * max_ctx + s of each cache array.
 *  paged:      token s of sequence b is row (block_table[b][s / page_size]) *
 *              page_size + s % page_size of each cache array. */
typedef struct {
  int32_t layout;              /* dsa_kv_layout_t                                       */
  int32_t batch;               /* B sequences                                           */
  int32_t max_ctx;             /* contiguous: token slots per sequence; paged: upper
                                  bound on every seqlen (<= max_pages * page_size)      */
  int32_t page_size;           /* paged only: tokens per page, a multiple of 64         */
  int32_t num_pages;           /* paged only: physical pages in the cache arrays        */
  int32_t max_pages;           /* paged only: columns of block_table                    */
  const int32_t* block_table;  /* paged only: device int32 [batch][max_pages]           */
  const int32_t* seqlens;      /* device int32 [batch]: tokens visible per sequence,
                                  including its query rows; NULL = max_ctx for all      */
} dsa_kv_desc_t;

/* Query rows. Each call processes the window of rows i in [row_begin,
 * row_begin + row_count) of every sequence (row_count = 0 means all rows from
 * row_begin through q_per_seq - 1); rows outside the window, and window rows a
 * sequence of a ragged batch does not have (i >= q_len[b]), are neither read nor
 * written. Score rows are stored compactly per window: window row i of sequence
 * b is score row b * row_count + (i - row_begin), whether or not the sequence
 * has that row. Indices, queries, outputs and LSE keep their global row
 * t = t0[b] + i.
 *
 * Ragged batches (q_start != NULL; the varlen layout of a batch of prompts of
 * different lengths, or of chunked-prefill pieces of different sizes, on one
 * cache, "dynamic KV cache" in the DSA principle section of the nsmao.com
 * report): sequence b owns the global rows [q_start[b], q_start[b + 1]), its
 * last q_len[b] = q_start[b + 1] - q_start[b] tokens (0 allowed). q_start is
 * device int32 [batch + 1], nondecreasing, q_start[0] >= 0, q_start[batch] <=
 * num_q, every q_len[b] <= q_per_seq and <= seqlen[b]; the kernels check these
 * and report DSA_ERR_BOUNDS through dsa_get_device_error for a sequence that
 * breaks them (its rows are then skipped). The host cannot read q_start, so
 * grids and score rows are sized for q_per_seq rows per sequence: choose it as
 * the largest q_len. */
typedef struct {
  int32_t num_q;               /* T: batch * q_per_seq (uniform), rows in q_start's
                                  range (ragged; at most batch * q_per_seq)             */
  int32_t q_per_seq;           /* query rows per sequence (>= 1); ragged: the largest  */
  int32_t row_begin;           /* first row of the window (0 = from the first row)      */
  int32_t row_count;           /* rows in the window (0 = through row q_per_seq - 1)    */
  const int32_t* q_start;      /* NULL (uniform), or device int32 [batch + 1] (ragged)  */
} dsa_q_desc_t;

/* Lightning-indexer scores (Eq. 1 of the report, FP8 as its §1 allows).
 *  q_idx   bf16 [T][64][128]  indexer queries; each (t, j) row is quantized on
 *                             the fly to E4M3 with scale s_q = max(amax, 2^-120)/448
 *  w       fp32 [T][64]       head weights w_{t,j}
 *  k_idx   uint8 E4M3 codes, [B][max_ctx][128] or paged [num_pages][page_size][128]
 *  k_scale fp32, [B][max_ctx] or paged [num_pages][page_size]: per-token key scale
 *  scores  fp32 [batch * row_count][ld] out (see dsa_q_desc_t for the row order):
 *                             scores[t][s] = s_k[s] * sum_j w_{t,j} s_q[t,j] *
 *                             ReLU(q_hat_{t,j} . k_hat_s) for s <= pos(t), -inf for
 *                             pos(t) < s < the end of the 128-key tile holding pos(t);
 *                             later columns are not written.
 *  ld      row stride of scores in elements, >= max_ctx rounded up to 128 and a
 *          multiple of 4. */
DSA_API dsa_status_t dsa_indexer_scores(const void* q_idx, const float* w, const void* k_idx,
                                const float* k_scale, const dsa_kv_desc_t* kv,
                                const dsa_q_desc_t* q, float* scores, int64_t ld,
                                dsa_stream_t stream);

/* Fine-grained token selection (report §1 and §2.1: S_t = Top-k(I_{t,:})).
 *  scores fp32 [batch * row_count][ld] as dsa_indexer_scores writes it: the
 *         row of query t is read on [0, pos(t)] only. 16-byte aligned, ld >= max_ctx
 *         and a multiple of 4.
 *  idx    int32 [T][k] out: the k highest-scoring positions of row t in
 *         ascending order; equal scores keep the lower position (-0.0 == +0.0);
 *         when pos(t) + 1 <= k all visible positions are selected and the rest
 *         of the row is -1. NaN scores are unsupported. */
DSA_API dsa_status_t dsa_topk(const float* scores, int64_t ld, const dsa_kv_desc_t* kv,
                      const dsa_q_desc_t* q, int32_t k, int32_t* idx, dsa_stream_t stream);

/* dsa_topk with a scratch buffer that lets long rows be swept by several CTAs at
 * once (the same selection, bit for bit). Rows of more than 4k visible keys are cut
 * into chunks of 16384 keys; each chunk's CTA keeps the keys at or above the row's
 * sample threshold (the one dsa_topk uses) as candidates, and one CTA per row then
 * selects the exact top k from the candidates, or from the whole row when the
 * candidates cannot decide it. Applies when max_ctx <= 131072; otherwise, or with a
 * workspace smaller than dsa_topk_workspace_size(), the call is dsa_topk.
 *  workspace  device, 256-byte aligned, or NULL; the library writes it during the
 *             call (stream order) and keeps nothing in it afterwards.
 * Other arguments as dsa_topk. */
DSA_API size_t dsa_topk_workspace_size(const dsa_kv_desc_t* kv, const dsa_q_desc_t* q, int32_t k);
DSA_API dsa_status_t dsa_topk_ws(const float* scores, int64_t ld, const dsa_kv_desc_t* kv,
                                 const dsa_q_desc_t* q, int32_t k, void* workspace,
                                 size_t workspace_bytes, int32_t* idx, dsa_stream_t stream);

/* Sparse MLA forward in MQA mode (report §1 Eq. 2, Fig. 1).
 *  q     bf16 [T][128][576] absorbed queries
 *  kv    bf16 latent cache, [B][max_ctx][576] or paged [num_pages][page_size][576]
 *  idx   int32 [T][k]: logical token positions; entries outside [0, pos(t)]
 *        (e.g. the -1 padding) are skipped; duplicates count as often as listed
 *  scale softmax scale applied to q . c_s
 *  out   bf16 [T][128][512] out: o_{t,h} = sum_s softmax_s(scale q_{t,h} . c_s) c_s[0:512]
 *  lse   fp32 [T][128] out: ln sum_s exp(scale q_{t,h} . c_s); a row with no
 *        valid entry gets o = 0 and lse = -inf. */
DSA_API dsa_status_t dsa_sparse_mla_fwd(const void* q, const void* kv_cache, const dsa_kv_desc_t* kv,
                                const dsa_q_desc_t* qd, const int32_t* idx, int32_t k,
                                float scale, void* out, float* lse, dsa_stream_t stream);

/* dsa_sparse_mla_fwd with a scratch buffer that lets the call balance its last wave.
 * The rows run as one 2-CTA cluster each, (SMs / 2) clusters at a time; when the
 * last wave would hold at most half as many rows as a full one, each of its rows is
 * split into 2..8 key segments (consecutive parts of its idx row, at least 288
 * entries each) run as clusters of their own, and a second kernel merges the
 * segments: LSE = ln sum_s e^{LSE_s}, o = sum_s e^{LSE_s - LSE} o_s. Results agree
 * with dsa_sparse_mla_fwd up to fp32 rounding (not bit for bit).
 *  workspace  device, 256-byte aligned, workspace_bytes long, or NULL / 0 (then no
 *             row is split and the call is dsa_sparse_mla_fwd). The library writes
 *             it during the call (stream order) and keeps nothing in it afterwards.
 *             Fewer bytes than dsa_sparse_mla_workspace_size() only allow fewer
 *             segments. Other arguments as dsa_sparse_mla_fwd. */
DSA_API dsa_status_t dsa_sparse_mla_fwd_ws(const void* q, const void* kv_cache,
                                           const dsa_kv_desc_t* kv, const dsa_q_desc_t* qd,
                                           const int32_t* idx, int32_t k, float scale,
                                           void* workspace, size_t workspace_bytes, void* out,
                                           float* lse, dsa_stream_t stream);

/* Bytes of scratch with which dsa_sparse_mla_fwd_ws may split every row it would
 * split on this device (at most (SMs / 2) segments of 256.5 KB). */
DSA_API size_t dsa_sparse_mla_workspace_size(void);

/* Indexer training target and KL loss term (report §2.1: the main attention summed
 * over all heads and L1-normalised along the sequence is the target p_{t,:}; the
 * indexer is trained with KL(p_{t,:} || Softmax(I_{t,:})), over every visible key in
 * the dense warm-up stage and over S_t in the sparse stage). For query row t and the
 * set S of entries of idx[t] inside [0, pos(t)] (as listed):
 *   a_h(s) = exp(scale q_{t,h} . c_s - lse[t][h])   (head h's attention over S)
 *   p(s)   = mean_h a_h(s),   q(s) = softmax_{s in S}(I_{t,s})
 *   kl[r]  = sum_{s in S} p(s) (ln p(s) - ln q(s))    (0 for an empty S)
 *  q, kv, the caches' geometry and idx as for dsa_sparse_mla_fwd; k in [1, 2^20]
 *         (the dense stage passes every visible position)
 *  lse    fp32 [T][128] the LSE dsa_sparse_mla_fwd wrote for the same idx and scale
 *  scores fp32 [batch * row_count][ld] indexer score rows of the window (as
 *         dsa_indexer_scores writes them); ld >= max_ctx
 *  kl     fp32 [batch * row_count] out, one term per row of the window.
 * A window row a ragged batch's sequence does not have gets kl = 0.
 * Shapes: 128 heads x 576-d latents only. */
DSA_API dsa_status_t dsa_indexer_kl(const void* q, const void* kv_cache, const dsa_kv_desc_t* kv,
                                    const dsa_q_desc_t* qd, const int32_t* idx, int32_t k,
                                    float scale, const float* lse, const float* scores,
                                    int64_t ld, float* kl, dsa_stream_t stream);

/* Bytes of device workspace dsa_forward needs for this geometry (0 on a
 * geometry the library rejects). */
DSA_API size_t dsa_workspace_size(const dsa_kv_desc_t* kv, const dsa_q_desc_t* q, int32_t k);

/* The whole forward: indexer scores -> top-k -> sparse MLA, on `stream`.
 * Arguments as in the three calls above. `workspace` (256-byte aligned) holds
 * the selected indices (unless idx_out is given) and one chunk of score rows;
 * dsa_workspace_size() bytes let the score rows go in chunks of up to 2 GiB. A
 * smaller workspace is accepted down to the indices plus one score row per
 * sequence; the rows are then processed in smaller chunks. Too small a
 * workspace returns DSA_ERR_WORKSPACE. The selection is dsa_topk's (one CTA per
 * row). Once the selection is done, the space of the
 * score rows serves the sparse MLA as dsa_sparse_mla_fwd_ws's scratch (split rows of
 * a partly filled last wave); dsa_workspace_size() includes what that needs.
 * idx_out (int32 [T][k]) receives the selection when not NULL. */
DSA_API dsa_status_t dsa_forward(const void* q_idx, const float* w, const void* k_idx,
                         const float* k_scale, const void* q, const void* kv_cache,
                         const dsa_kv_desc_t* kv, const dsa_q_desc_t* qd, int32_t k,
                         float scale, void* workspace, size_t workspace_bytes,
                         int32_t* idx_out, void* out, float* lse, dsa_stream_t stream);

/* dsa_forward without a workspace argument, for callers that cannot allocate
 * device memory themselves: for example a plugin that its host framework hands
 * only input and output buffers, or a runtime whose device memory all belongs
 * to its own pool allocator, so that neither cudaMalloc nor a framework
 * allocator may be called for scratch space. (The technical report has no
 * counterpart of this call; it is an interface convenience.)
 *  - The scratch space is a fixed 128 MiB device array inside this library;
 *    every GPU that loads the library holds it until the process exits. The
 *    call allocates nothing.
 *  - It must hold the selected indices (T * k * 4 bytes, none when idx_out is
 *    given) plus at least one score row per sequence (round_up(max_ctx, 128) * 4
 *    * batch bytes); larger geometries return DSA_ERR_WORKSPACE before anything
 *    is launched. Score rows are processed in chunks that fit.
 *  - The first call on each device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture begins.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents (nothing in it needs to start at zero). Calls whose kernels
 *    overlap on the GPU, e.g. on two streams at once, race on it: serialize them.
 * Arguments and results are those of dsa_forward. */
DSA_API dsa_status_t dsa_forward_noalloc(const void* q_idx, const float* w, const void* k_idx,
                                         const float* k_scale, const void* q,
                                         const void* kv_cache, const dsa_kv_desc_t* kv,
                                         const dsa_q_desc_t* qd, int32_t k, float scale,
                                         int32_t* idx_out, void* out, float* lse,
                                         dsa_stream_t stream);

/* ---- Fused indexer -> top-k: the selection without stored score rows ------------------
 * The same selection as dsa_indexer_scores + dsa_topk (report §1 and §2.1: S_t =
 * Top-k(I_{t,:}); equal scores keep the lower position, ascending, -1 padded),
 * without ever writing a row's scores to memory:
 *   1. a strided pass scores every 8th 128-key tile of each row and takes the m-th
 *      largest of that sample as the row's threshold (m = k/8 + 6 sqrt(k/8) + 32,
 *      so the threshold lies well below the row's k-th score);
 *   2. a second pass scores every key and keeps, per row, the keys at or above the
 *      threshold as candidates (at most cand_cap per row);
 *   3. the exact top-k of the candidates is selected. A row whose candidates are
 *      fewer than k or more than cand_cap cannot be decided from them; such rows
 *      (rare) are selected from their full score rows, so the result is always
 *      identical to dsa_indexer_scores + dsa_topk.
 * The call synchronizes `stream` once per chunk of rows to read the count of such
 * rows. Requires max_ctx <= 131072.
 *  cand_cap  candidates kept per row, 0 = 8192 (the most); smaller values force the
 *            full-row path more often (a test hook)
 *  workspace 256-byte aligned, dsa_fused_workspace_size() bytes for the largest chunk
 *            of rows; smaller workspaces (down to one row per sequence) take smaller
 *            chunks
 *  idx       int32 [T][k] out, as dsa_topk writes it. */
DSA_API size_t dsa_fused_workspace_size(const dsa_kv_desc_t* kv, const dsa_q_desc_t* q,
                                        int32_t k);
DSA_API dsa_status_t dsa_select_fused(const void* q_idx, const float* w, const void* k_idx,
                                      const float* k_scale, const dsa_kv_desc_t* kv,
                                      const dsa_q_desc_t* qd, int32_t k, int32_t cand_cap,
                                      void* workspace, size_t workspace_bytes, int32_t* idx,
                                      dsa_stream_t stream);

/* dsa_forward with the fused selection: dsa_select_fused then dsa_sparse_mla_fwd_ws.
 * Arguments as dsa_forward plus cand_cap; the workspace holds the indices (unless
 * idx_out is given) followed by dsa_select_fused's workspace, which then serves as
 * the sparse MLA's split scratch (dsa_fused_workspace_size() includes what that
 * needs). */
DSA_API dsa_status_t dsa_forward_fused(const void* q_idx, const float* w, const void* k_idx,
                                       const float* k_scale, const void* q,
                                       const void* kv_cache, const dsa_kv_desc_t* kv,
                                       const dsa_q_desc_t* qd, int32_t k, float scale,
                                       int32_t cand_cap, void* workspace, size_t workspace_bytes,
                                       int32_t* idx_out, void* out, float* lse,
                                       dsa_stream_t stream);

/* ---- MLA in MHA mode: the masked-MHA emulation of DSA for short prefill ----------
 * Report Appendix A (Fig. 4): MLA runs in an MHA mode (training, prefill) or an MQA
 * mode (decode); report §3 "Inference cost": for short-sequence prefill a masked MHA
 * mode emulates DSA. Per head h (128 heads) the MHA-mode key of token s is
 * k_{h,s} = [W^UK_h c_s[0:512] ; c_s[512:576]] (128 nope dims, then the 64 rope
 * dims every head shares) and its value v_{h,s} = W^UV_h c_s[0:512] (128 dims);
 * the query of row t is q_{t,h} = [q^C (128) ; q^R (64)]. Row t attends over its
 * selected set S_t (every visible key when pos(t) + 1 <= k): the result equals
 * the MQA-mode sparse MLA of the absorbed query [W^UK_h^T q^C ; q^R] followed by
 * W^UV_h on its output, with the same LSE. */

/* Decompresses the latent cache into MHA-mode keys and values (bf16, fp32
 * accumulation). For every sequence b, head h and token s < seqlen[b]:
 *  k_nope bf16 [batch][128][ctx_pad][128] out: W^UK_h c_s[0:512]
 *  k_rope bf16 [batch][ctx_pad][64]      out: c_s[512:576]
 *  v      bf16 [batch][128][ctx_pad][128] out: W^UV_h c_s[0:512]
 * Slots s in [seqlen, round_up(seqlen, 128)) are written as zeros; later slots are
 * not written.
 *  kv_cache bf16 latent cache as for dsa_sparse_mla_fwd (contiguous or paged)
 *  w_uk, w_uv bf16 [128][128][512]: row d of head h is the weight vector of output
 *           dim d (W^UK_h and W^UV_h, row-major)
 *  ctx_pad  a multiple of 128, >= max_ctx rounded up to 128; batch * 128 * ctx_pad
 *           must stay below 2^31. */
DSA_API dsa_status_t dsa_mla_up_project(const void* kv_cache, const void* w_uk, const void* w_uv,
                                        const dsa_kv_desc_t* kv, void* k_nope, void* k_rope,
                                        void* v, int64_t ctx_pad, dsa_stream_t stream);

/* Selection bitmask of the window's rows: for every row t of the window with
 * pos(t) + 1 > k, bit s of mask[t] (word s / 32, bit s % 32) is set iff s is an
 * entry of idx[t] inside [0, pos(t)]; the words of the 128-key tiles up to pos(t)
 * are written, the rest of the row is not. Rows with pos(t) + 1 <= k select every
 * visible key and are not written.
 *  idx  int32 [T][k] (as dsa_topk writes it)
 *  mask uint32 [T][mask_ld] out, 16-byte aligned; mask_ld a multiple of 4 and
 *       >= 4 * ceil(max_ctx / 128) (at most 58112 words). */
DSA_API dsa_status_t dsa_selection_mask(const int32_t* idx, int32_t k, const dsa_kv_desc_t* kv,
                                        const dsa_q_desc_t* qd, uint32_t* mask, int64_t mask_ld,
                                        dsa_stream_t stream);

/* Masked MHA over the decompressed keys and values (flash attention, 128-row by
 * 128-key tiles on the tensor cores, P rounded to bf16):
 *  q_mha bf16 [T][128][192] MHA-mode queries (128 nope dims, then 64 rope dims)
 *  k_nope, k_rope, v, ctx_pad as dsa_mla_up_project wrote them
 *  mask  NULL: every row attends over all of 0..pos(t) (causal MHA). Otherwise
 *        rows with pos(t) + 1 > k attend over the keys whose bit is set in
 *        mask[t] (dsa_selection_mask), the others over 0..pos(t).
 *  out   bf16 [T][128][128] out: o_{t,h} = sum_s softmax_s(scale q_{t,h} . k_{h,s}) v_{h,s}
 *  lse   fp32 [T][128] out: ln sum_s exp(scale q_{t,h} . k_{h,s}); a row with no
 *        admitted key gets o = 0 and lse = -inf. */
DSA_API dsa_status_t dsa_masked_mha(const void* q_mha, const void* k_nope, const void* k_rope,
                                    const void* v, int64_t ctx_pad, const dsa_kv_desc_t* kv,
                                    const dsa_q_desc_t* qd, const uint32_t* mask,
                                    int64_t mask_ld, int32_t k, float scale, void* out,
                                    float* lse, dsa_stream_t stream);

/* Bytes of device workspace dsa_mha_prefill needs (0 on a rejected geometry). */
DSA_API size_t dsa_mha_workspace_size(const dsa_kv_desc_t* kv, const dsa_q_desc_t* q, int32_t k);

/* Short-prefill DSA in MHA mode: indexer scores and top-k for the rows with more
 * than k visible keys (when seqlens and q_start are NULL the rows with pos(t) + 1
 * <= k are skipped; otherwise every row of the window is scored), their
 * selection masks, the up-projection of the latent cache, then the masked MHA.
 * Inputs as for dsa_forward plus q_mha, w_uk and w_uv; out and lse as for
 * dsa_masked_mha. `workspace` (256-byte aligned) holds the indices (unless idx_out
 * is given), the masks, the decompressed keys and values and a chunk of score
 * rows; dsa_mha_workspace_size() bytes give the largest chunk, smaller
 * workspaces down to one score row per sequence are accepted. idx_out, when not
 * NULL, receives the selection of every row of the window. */
DSA_API dsa_status_t dsa_mha_prefill(const void* q_idx, const float* w, const void* k_idx,
                                     const float* k_scale, const void* q_mha,
                                     const void* kv_cache, const void* w_uk, const void* w_uv,
                                     const dsa_kv_desc_t* kv, const dsa_q_desc_t* qd, int32_t k,
                                     float scale, void* workspace, size_t workspace_bytes,
                                     int32_t* idx_out, void* out, float* lse,
                                     dsa_stream_t stream);

/* Synchronizes `stream`, then returns and clears the device error word
 * (DSA_OK when no kernel reported a problem since the last call). */
DSA_API dsa_status_t dsa_get_device_error(dsa_stream_t stream);

/* Upper bound, in nanoseconds, on every bounded device-side wait (default
 * 2e9). Returns the previous value. A value of 0 restores the default. */
DSA_API uint64_t dsa_set_wait_timeout_ns(uint64_t ns);

/* Launches one kernel whose bounded wait can never be satisfied, so that the
 * timeout path is exercised without a fault: returns DSA_ERR_DEVICE_TIMEOUT
 * (after about the configured timeout) when the path works. */
DSA_API dsa_status_t dsa_selftest_wait_timeout(dsa_stream_t stream);

/* Static description of a status code. */
DSA_API const char* dsa_status_string(dsa_status_t status);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* DSA_H_ */
