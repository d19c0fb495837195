// Work planning on the device (one CTA), so no length ever travels to the host.
//
// Reads query_start_loc and seq_lens, sanitises them into SeqInfo, and builds
//  - the prefill work list: one entry per 256-query-row item (two 128-row
//    tiles) of every sequence with more than one query, with the KV tiles
//    each tile visits (causal, full-attention spans, or all keys), ordered
//    by descending KV-tile count (longest work first, for the persistent
//    prefill grid);
//  - the exclusive prefix of 16-key pages over the single-query (decode)
//    sequences, from which the decode CTAs cut their balanced page ranges
//    when there are too many sequences for them to plan themselves;
//  - zeroed split-KV arrival counters;
//  - when the call runs its prefill and decode kernels side by side, the
//    share of the SMs each gets, from a cost model of the two kinds of work
//    (prefill tile visits against decode bytes; see split_machine).
// This plays the role of the device-side runtime length reduction of
// ROCm/TransformerEngine PR #461 (description: the real maximum is found on
// the device before routing), without any host synchronisation.
#include "common.cuh"
#include "kernels.h"
#include "layout.h"
#include "spans.cuh"

namespace pa {

namespace {

constexpr int kPlanThreads = 1024;

// Block-wide exclusive scan of one int per thread; returns the block total.
__device__ int block_exclusive_scan(int v, int* out_excl, int* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < (int)(blockDim.x >> 5)) ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_warp[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  int warp_prefix = warp ? s_warp[warp - 1] : 0;
  *out_excl = warp_prefix + x - v;
  int total = s_warp[(blockDim.x >> 5) - 1];
  __syncthreads();
  return total;
}

// KV tiles of one 128-row tile whose rows are [row0, row0 + rows): enough
// for the most keys any of its rows sees (causal, spans or neither)
__device__ __forceinline__ int kv_tiles(const SeqInfo& si, int row0, int rows, int causal,
                                        const SpanList& sl, bool* malformed) {
  if (rows <= 0) return 0;
  int vis = si.kv_len;
  const int p0 = si.kv_len - si.q_len + row0;  // key positions of the tile's rows
  if (sl.pairs || !sl.offsets_ok)
    vis = span_visible(sl, p0, p0 + rows - 1, malformed);
  else if (causal)
    vis = max(0, min(si.kv_len, p0 + rows));
  return (vis + kPrefillTileN - 1) / kPrefillTileN;
}

// KV tiles of a 256-row work item's two 128-row tiles
__device__ __forceinline__ int2 item_tiles(const SeqInfo& si, int row0, int causal,
                                           const SpanList& sl, bool* malformed) {
  const int rows_a = min(kPrefillTileM, si.q_len - row0);
  const int rows_b = min(kPrefillTileM, si.q_len - row0 - kPrefillTileM);
  bool bad_a = false, bad_b = false;
  const int2 n = make_int2(kv_tiles(si, row0, rows_a, causal, sl, &bad_a),
                           kv_tiles(si, row0 + kPrefillTileM, rows_b, causal, sl, &bad_b));
  if (malformed) *malformed = bad_a || bad_b;
  return n;
}

// The SMs the prefill and the decode kernel each use when they run side by
// side on split.sms SMs (both 0 when split.sms is 0: one after the other, each
// on the whole machine).  With only one kind of work, each may take every SM.
// Otherwise the prefill gets the P SMs that minimise the later finish time:
// the prefill's work spread over P SMs, against the decode's bytes streamed by
// the other SMs at no more than kDecodeSmBytesPerUs each and
// kDecodeHbmBytesPerUs in all.  Called by one whole warp: each lane tries
// every 32nd P, then the warp keeps the best (the smallest P on a tie).
__device__ int2 split_machine(const SplitShape& split, float visits, float pages) {
  if (split.sms <= 1) return make_int2(0, 0);
  const float wp = visits * split.num_q_heads * (float)kPrefillTileVisitUs * split.head_dim / 128.f;
  const float bytes = pages * kPageKeys * split.num_kv_heads * split.head_dim * 4.f;
  if (!(wp > 0.f) || !(bytes > 0.f)) return make_int2(split.sms, split.sms);
  const float t_hbm = bytes / (float)kDecodeHbmBytesPerUs;
  float best_t = INFINITY;
  int best_p = split.sms;
  for (int p = 1 + (threadIdx.x & 31); p < split.sms; p += 32) {
    const float t = fmaxf(wp / p, fmaxf(bytes / ((split.sms - p) * (float)kDecodeSmBytesPerUs), t_hbm));
    if (t < best_t) {
      best_t = t;
      best_p = p;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ot = __shfl_xor_sync(0xffffffffu, best_t, o);
    const int op = __shfl_xor_sync(0xffffffffu, best_p, o);
    if (ot < best_t || (ot == best_t && op < best_p)) {
      best_t = ot;
      best_p = op;
    }
  }
  if (best_p >= split.sms) best_p = split.sms / 2;
  return make_int2(best_p, split.sms - best_p);
}

}  // namespace

__global__ void __launch_bounds__(kPlanThreads, 1)
    plan_kernel(const int32_t* __restrict__ query_start_loc, const int32_t* __restrict__ seq_lens,
                int num_seqs, long long num_q_tokens, int max_blocks_per_seq, int block_size,
                int max_query_len, int max_seq_len, int causal, long long num_counters,
                const int32_t* __restrict__ span_offsets, const int32_t* __restrict__ spans,
                int num_spans, unsigned char* ws, WorkspaceLayout L, SplitShape split) {
  uint32_t* err = reinterpret_cast<uint32_t*>(ws + L.err);
  PlanHeader* hdr = reinterpret_cast<PlanHeader*>(ws + L.header);
  SeqInfo* info = reinterpret_cast<SeqInfo*>(ws + L.seq_info);
  int2* tiles = reinterpret_cast<int2*>(ws + L.tiles);
  int2* tile_n = reinterpret_cast<int2*>(ws + L.tile_n);
  int32_t* page_pfx = reinterpret_cast<int32_t*>(ws + L.page_pfx);
  int32_t* counters = reinterpret_cast<int32_t*>(ws + L.counters);

  __shared__ int s_warp[32];
  __shared__ int s_hist[kCostBuckets];
  __shared__ int s_carry;
  __shared__ uint32_t s_err;
  __shared__ float s_visits;  // prefill tile visits (128-row tile x KV tile), summed per warp

  const int tid = threadIdx.x;
  if (tid == 0) {
    s_err = 0;
    s_visits = 0.f;
  }
  for (int i = tid; i < kCostBuckets; i += blockDim.x) s_hist[i] = 0;
  for (long long i = tid; i < num_counters; i += blockDim.x) counters[i] = 0;
  __syncthreads();

  // ---- pass 1: sanitise lengths, total decode keys -------------------------
  const long long reach = (long long)max_blocks_per_seq * block_size;
  for (int s = tid; s < num_seqs; s += blockDim.x) {
    uint32_t e = 0;
    long long qs = query_start_loc[s], qe = query_start_loc[s + 1];
    long long kv = seq_lens[s];
    if (qs < 0 || qe < qs || qe > num_q_tokens) {
      e |= PA_DEVERR_LENGTHS;
      qe = qs = max(0ll, min(qs, num_q_tokens));
    }
    if (kv < 0) {
      e |= PA_DEVERR_LENGTHS;
      kv = 0;
    }
    if (kv > reach) {
      e |= PA_DEVERR_LENGTHS;
      kv = reach;
    }
    long long ql = qe - qs;
    if (ql > kv) e |= PA_DEVERR_QLEN;
    if (ql > max_query_len || kv > max_seq_len) e |= PA_DEVERR_HINT;
    SeqInfo si;
    si.q_start = (int)qs;
    si.q_len = (int)ql;
    si.kv_len = (int)kv;
    si.pad = 0;
    info[s] = si;
    if (e) atomicOr(&s_err, e);
  }
  __syncthreads();

  // ---- pass 2: decode page prefix, tile histogram --------------------------
  if (tid == 0) s_carry = 0;
  __syncthreads();
  int my_visits = 0;  // this thread's prefill tile visits
  for (int base = 0; base < num_seqs; base += blockDim.x) {
    const int s = base + tid;
    int pages = 0;
    if (s < num_seqs) {
      const SeqInfo si = info[s];
      if (si.q_len == 1) pages = (si.kv_len + kPageKeys - 1) / kPageKeys;
      if (si.q_len > 1) {
        const SpanList sl = span_list(span_offsets, spans, num_spans, s, si.kv_len);
        bool bad = false;
        for (int r = 0; r < si.q_len; r += kPrefillItemRows) {
          bool bad_r = false;
          const int2 n = item_tiles(si, r, causal, sl, &bad_r);
          bad |= bad_r;
          const int c = n.x + n.y;
          atomicAdd(&s_hist[kCostBuckets - 1 - min(c, kCostBuckets - 1)], 1);
          my_visits += c;
        }
        if (bad) atomicOr(&s_err, PA_DEVERR_SPANS);
      }
    }
    int excl;
    const int total = block_exclusive_scan(pages, &excl, s_warp);
    if (s < num_seqs) page_pfx[s] = s_carry + excl;
    __syncthreads();
    if (tid == 0) s_carry += total;
    __syncthreads();
  }
  if (tid == 0) page_pfx[num_seqs] = s_carry;
  const int total_pages = s_carry;
  {
    float v = (float)my_visits;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((tid & 31) == 0 && v > 0.f) atomicAdd(&s_visits, v);
  }

  // ---- pass 3: counting sort of prefill tiles by descending cost -----------
  // exclusive scan of the histogram (bucket 0 = most expensive)
  {
    constexpr int per = kCostBuckets / kPlanThreads;
    int local[per];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) {
      local[i] = s_hist[tid * per + i];
      sum += local[i];
    }
    int excl;
    block_exclusive_scan(sum, &excl, s_warp);
#pragma unroll
    for (int i = 0; i < per; ++i) {
      s_hist[tid * per + i] = excl;
      excl += local[i];
    }
  }
  __syncthreads();
  int num_tiles = 0;
  for (int s = tid; s < num_seqs; s += blockDim.x) {
    SeqInfo si = info[s];
    if (si.q_len > 1) {
      const SpanList sl = span_list(span_offsets, spans, num_spans, s, si.kv_len);
      for (int r = 0; r < si.q_len; r += kPrefillItemRows) {
        const int2 n = item_tiles(si, r, causal, sl, nullptr);
        const int c = n.x + n.y;
        int pos = atomicAdd(&s_hist[kCostBuckets - 1 - min(c, kCostBuckets - 1)], 1);
        if ((long long)pos < (long long)L.max_tiles) {  // overlapping query ranges can overflow
          tiles[pos] = make_int2(s, r);
          tile_n[pos] = n;
        } else {
          atomicOr(&s_err, PA_DEVERR_LENGTHS);
        }
      }
    }
  }
  __syncthreads();
  if (tid < 32) {
    const int2 sms = split_machine(split, s_visits, (float)total_pages);
    if (tid == 0) {
      hdr->prefill_sms = sms.x;
      hdr->decode_sms = sms.y;
    }
  }
  if (tid == 0) {
    // the last bucket's running cursor ends at the number of tiles
    num_tiles = (int)min((long long)s_hist[kCostBuckets - 1], (long long)L.max_tiles);
    hdr->num_prefill_tiles = num_tiles;
    hdr->total_decode_pages = total_pages;
    hdr->prefill_next = 0;
    if (s_err) atomicOr(err, s_err);
  }
}

void launch_plan(const int32_t* query_start_loc, const int32_t* seq_lens, int num_seqs,
                 long long num_q_tokens, int max_blocks_per_seq, int block_size,
                 int max_query_len, int max_seq_len, int causal, long long num_counters,
                 const int32_t* span_offsets, const int32_t* spans, int num_spans,
                 unsigned char* ws, const WorkspaceLayout& L, const SplitShape& split,
                 cudaStream_t stream) {
  plan_kernel<<<1, kPlanThreads, 0, stream>>>(query_start_loc, seq_lens, num_seqs, num_q_tokens,
                                              max_blocks_per_seq, block_size, max_query_len,
                                              max_seq_len, causal, num_counters, span_offsets,
                                              spans, num_spans, ws, L, split);
}

}  // namespace pa
