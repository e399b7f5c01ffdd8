// The sequence a prefill work unit belongs to: its query count, its key count
// and where its rows start, for the padded layout ([B, nh, S, hd] queries over
// a [B, nkv, cap, hd] cache) and the packed variable-length layout (the
// sequences of a batch concatenated along the token axis, delimited by
// cumulative offsets, as the FlashAttention-3 summary's variable-length
// sequences are read).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace gqa {

struct SeqRange {
  int S;        // query rows of the sequence
  int kv_len;   // keys of the sequence
  int q0, k0;   // packed: first query / key row of the sequence (0 when padded)
};

// Offsets and lengths are clamped to the tensors the caller passed; a clamp,
// or a packed query run longer than the caller's longest (p.S, which sizes
// the grid: rows past the grid are not written), is recorded in the device
// error word (by one thread per CTA).
__device__ __forceinline__ SeqRange prefill_seq(const PrefillParams& p, int b, int* err) {
  SeqRange r;
  bool bad = false;
  if (p.cu_q) {
    const int q_lo = p.cu_q[b], q_hi = p.cu_q[b + 1], k_lo = p.cu_k[b], k_hi = p.cu_k[b + 1];
    r.q0 = min(max(q_lo, 0), p.total_q);
    r.k0 = min(max(k_lo, 0), p.cap);
    const int q_end = min(max(q_hi, r.q0), p.total_q), k_end = min(max(k_hi, r.k0), p.cap);
    r.S = q_end - r.q0;
    r.kv_len = k_end - r.k0;
    bad = r.q0 != q_lo || q_end != q_hi || r.k0 != k_lo || k_end != k_hi || r.S > p.S;
    if (bad && threadIdx.x == 0) raise_error(err, GQA_DEVERR_SEQLEN_RANGE);
  } else {
    r.S = p.S;
    r.q0 = r.k0 = 0;
    r.kv_len = p.kv_lens[b];
    if (r.kv_len > p.cap || r.kv_len < 0) {
      if (threadIdx.x == 0) raise_error(err, GQA_DEVERR_KVLEN_RANGE);
      r.kv_len = r.kv_len > p.cap ? p.cap : 0;
    }
  }
  return r;
}

}  // namespace gqa
