// rows.cuh -- where each query row sits: its sequence, its global row index and
// its causal position.
//
// The query rows of sequence b are its last q_len tokens (decode: the 1 or 2
// newest tokens; prefill: the whole prompt; chunked prefill: the chunk appended
// after the tokens already cached, "dynamic KV cache" in the DSA principle
// section of "DeepSeek-V3.2开源技术报告"). Row i of the sequence (0 <= i < q_len)
// is global row t0 + i and sees the keys s <= pos = seqlen - q_len + i.
//   uniform batch (q_start == nullptr): t0 = b * q_per_seq, q_len = q_per_seq
//   ragged batch:                        t0 = q_start[b], q_len = q_start[b+1] - q_start[b]
// q_per_seq bounds every q_len; a sequence whose rows or length are out of range
// has ok = false (the caller reports it and skips the sequence; in a uniform batch
// t0 and q_len still name its rows).
#pragma once

#include <cstdint>

namespace dsa {

struct SeqRows {
  int64_t t0;  // global row of the sequence's first query row
  int q_len;   // query rows of the sequence
  int seqlen;  // visible tokens of the sequence, its query rows included
  bool ok;     // rows and length in range
};

__device__ __forceinline__ SeqRows seq_rows(const int32_t* q_start, const int32_t* seqlens, int b,
                                            int q_per_seq, int num_q, int max_ctx) {
  SeqRows r;
  r.seqlen = seqlens ? __ldg(seqlens + b) : max_ctx;
  if (q_start) {
    const int a = __ldg(q_start + b), e = __ldg(q_start + b + 1);
    r.t0 = a;
    r.q_len = e - a;
    r.ok = a >= 0 && e <= num_q && r.q_len >= 0 && r.q_len <= q_per_seq;
    if (!r.ok) r.q_len = 0;
  } else {
    r.t0 = (int64_t)b * q_per_seq;
    r.q_len = q_per_seq;
    r.ok = true;
  }
  r.ok = r.ok && r.seqlen >= r.q_len && r.seqlen <= max_ctx;
  return r;
}

}  // namespace dsa
