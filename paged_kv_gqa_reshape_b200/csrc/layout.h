// Workspace layout and per-call work plan shared by the host API and the
// kernels.  Everything here is sized from call arguments only, so the host
// can size the workspace without touching the device.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace pa {

constexpr int kPrefillTileM = 128;      // query rows per prefill tile (tcgen05 M)
constexpr int kPrefillItemRows = 256;   // query rows per prefill work item: two tiles
constexpr int kPrefillTileN = 128;      // keys per prefill KV tile (tcgen05 N)
constexpr int kPageKeys = 16;           // keys per page: the unit the kernels fetch and count
constexpr int kMaxBlockSize = 512;      // block_size: a power of two from kPageKeys up to this

// log2 of the 16-key pages in a cache block of block_size slots (a power of two >= 16).
inline int log2_pages_per_block(int block_size) {
  int s = 0;
  while ((kPageKeys << s) < block_size) ++s;
  return s;
}
constexpr int kDecodeMaxWarps = 4096;   // bound on decode warps in one launch (8 per SM)
constexpr int kCostBuckets = 4096;      // prefill tiles are sorted by KV-tile count
constexpr int kSelfPlanMaxSeqs = 1024;  // decode CTAs plan for themselves up to this many sequences
// Split-KV arrival counters live at a fixed offset, in a region no layout
// uses for anything else, at least this many int32 long.  Each merge resets
// its counter after use, so once the workspace has been zeroed the region
// stays zero between calls whatever their sizes; a call that plans for itself
// (no plan kernel to zero them) must fit its counters in this region.
constexpr int kFixedCounterSlots = 65536;

constexpr int kMaxGroup = 128;          // largest GQA group (num_q_heads / num_kv_heads)

// Warps of the decode kernel that share one KV head: one warp serves up to 16
// query heads of its GQA group, so larger groups are cut into 16-head slices;
// a power of two (1, 2, 4 or 8) so that the slices tile a CTA's warps.
inline int decode_slices(int64_t group) {
  int s = 1;
  while (s * 16 < group) s *= 2;
  return s;
}

// Sanitised geometry of one sequence, written by the plan kernel.  The
// attention kernels read lengths only from here, never from the raw inputs.
struct SeqInfo {
  int32_t q_start;    // first query token of the sequence
  int32_t q_len;      // number of query tokens (0 if the sequence is skipped)
  int32_t kv_len;     // number of keys (clamped to the block table's reach)
  int32_t pad;
};

struct PlanHeader {
  int32_t num_prefill_tiles;   // entries in the prefill tile list
  int32_t total_decode_pages;  // 16-key pages over all single-query sequences
  int32_t prefill_next;        // prefill work items handed out after the first round
  // When the prefill and decode kernels of a call run side by side, the SMs
  // each may use (the plan's split of the machine; see plan.cu)
  int32_t prefill_sms;
  int32_t decode_sms;
  int32_t pad[59];
};

// Cost model of the side-by-side split, measured on B200 at 1965 MHz:
// a prefill work item's 128-row tile visiting one 128-key KV tile of one head
// costs about kPrefillTileVisitUs SM-microseconds at head_dim 128 (prefill
// time x SMs / tile visits on the varlen and mixed-step workloads: 1.14 and
// 1.20); a decode CTA streams at most kDecodeSmBytesPerUs bytes per
// microsecond (about 59 GB/s per SM alone, from runs on 24 to 96 SMs; 56 GB/s
// beside the prefill, from the mixed step's 17 GB on 105 SMs in 2.90 ms), and
// the decode kernel as a whole at most kDecodeHbmBytesPerUs (7.2 TB/s, the
// mixed step's 17 GB of decode reads on all SMs).
constexpr double kPrefillTileVisitUs = 1.15;
constexpr double kDecodeSmBytesPerUs = 56.0e3;
constexpr double kDecodeHbmBytesPerUs = 7.2e6;

struct WorkspaceLayout {
  size_t err;        // uint32 error word (PA_ERROR_WORD_BYTES reserved)
  size_t header;     // PlanHeader
  size_t seq_info;   // SeqInfo[num_seqs]
  size_t tiles;      // int2[max_tiles]   (seq, first query row of a 256-row work item)
  size_t tile_n;     // int2[max_tiles]   KV tiles its two 128-row query tiles visit
  size_t page_pfx;   // int32[num_seqs + 1]  exclusive prefix of decode pages
  size_t counters;   // int32[max(num_seqs * num_kv_heads * slices, kFixedCounterSlots)]
                     // split-KV arrival counters, at a fixed offset (see kFixedCounterSlots)
  size_t lse;        // float[max_slots * num_q_heads]   log2-sum-exp per partial
  size_t partial;    // float[max_slots * num_q_heads * head_dim]
  size_t total;
  int64_t max_tiles;
  int64_t max_slots;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Split-KV arrival counters a call uses: one per (sequence, KV head, slice).
inline int64_t counter_slots_needed(int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads) {
  return num_seqs * num_kv_heads * decode_slices(num_q_heads / num_kv_heads);
}

inline WorkspaceLayout make_layout(int64_t num_seqs, int64_t num_q_tokens, int64_t num_q_heads,
                                   int64_t num_kv_heads, int64_t head_dim) {
  WorkspaceLayout L{};
  size_t off = 0;
  L.err = off;
  off += 256;
  L.header = off;
  off += sizeof(PlanHeader);
  L.counters = off;  // fixed offset: the same in every layout
  const int64_t need = counter_slots_needed(num_seqs, num_q_heads, num_kv_heads);
  const int64_t counter_slots = need > kFixedCounterSlots ? need : (int64_t)kFixedCounterSlots;
  off = align_up(off + 4 * (size_t)counter_slots, 256);
  L.seq_info = off;
  off = align_up(off + sizeof(SeqInfo) * (size_t)num_seqs, 256);
  L.max_tiles = (num_q_tokens + kPrefillItemRows - 1) / kPrefillItemRows + num_seqs;
  L.tiles = off;
  off = align_up(off + 8 * (size_t)L.max_tiles, 256);
  L.tile_n = off;
  off = align_up(off + 8 * (size_t)L.max_tiles, 256);
  // Decode CTA c of a KV-head group covering sequence s writes partial slot
  // c + s; a launch has at most kDecodeMaxWarps / Hkv page ranges per group.
  L.max_slots = (kDecodeMaxWarps + num_kv_heads - 1) / num_kv_heads + num_seqs;
  L.page_pfx = off;
  off = align_up(off + 4 * (size_t)(num_seqs + 1), 256);
  L.lse = off;
  off = align_up(off + 4 * (size_t)(L.max_slots * num_q_heads), 256);
  L.partial = off;
  off = align_up(off + 4 * (size_t)(L.max_slots * num_q_heads * head_dim), 256);
  L.total = off;
  return L;
}

}  // namespace pa
