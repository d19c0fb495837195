// Piecewise block-causal masking: full-attention spans inside causal
// sequences (vllm-omni PR #9244 "Support piecewise block-causal attention for
// full_attn_spans", description: the shared segment plan).  A query at key
// position p inside a used span [start, end) sees keys 0 .. end-1 (the
// truncated prefix, bidirectionally); any other query sees keys 0 .. p.
//
// Sequence s owns the (start, end) pairs spans[2k], spans[2k + 1] for k in
// [offsets[s], offsets[s + 1]).  A pair is used iff 0 <= start < end <= Lkv and
// start >= the previous pair's end; offsets outside [0, num_spans] or
// decreasing leave the sequence without spans.  The plan kernel (which raises
// PA_DEVERR_SPANS) and the prefill kernel apply the same rule.
#pragma once

#include <stdint.h>

namespace pa {

struct SpanList {
  const int32_t* pairs = nullptr;  // 2 * n ints
  int n = 0;
  int kv_len = 0;
  bool offsets_ok = true;
};

__device__ __forceinline__ SpanList span_list(const int32_t* offsets, const int32_t* spans,
                                              int num_spans, int seq, int kv_len) {
  SpanList L;
  L.kv_len = kv_len;
  if (!offsets) return L;
  const int a = offsets[seq], b = offsets[seq + 1];
  if (a < 0 || b < a || b > num_spans) {
    L.offsets_ok = false;
    return L;
  }
  L.pairs = spans + 2 * (size_t)a;
  L.n = b - a;
  return L;
}

// Visible keys (a prefix length) of the queries at key positions [p0, p1]:
// the largest over the range.  Also reports whether any pair is malformed.
__device__ __forceinline__ int span_visible(const SpanList& L, int p0, int p1, bool* malformed) {
  long long n = (long long)p1 + 1;
  int prev_end = 0;
  bool bad = false;
  for (int k = 0; k < L.n; ++k) {
    const int a = L.pairs[2 * k], e = L.pairs[2 * k + 1];
    const bool used = a >= 0 && a < e && e <= L.kv_len && a >= prev_end;
    bad |= !used;
    prev_end = e;
    if (used && a <= p1 && e > p0 && e > n) n = e;
  }
  if (malformed) *malformed = bad || !L.offsets_ok;
  if (n < 0) n = 0;
  if (n > L.kv_len) n = L.kv_len;
  return (int)n;
}

}  // namespace pa
