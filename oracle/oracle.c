/*
 * Reference oracle for paged KV attention — TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and the cpu_baseline leg of bench.py
 * may load this library.  The product path (the CUDA library and its Python
 * binding) never calls it and shares no code with it.
 *
 * Plain C, double precision, no blocking, no fusion, no reordering beyond
 * what the definitions state.  Every input element is a bfloat16 bit pattern
 * (uint16_t) widened exactly to double; every result is a double.
 *
 * What it computes, and where the definition comes from:
 *
 *  oracle_write_kv
 *      The cache write of vllm-spyre PR #853 "Pytorch Native Attention on
 *      Spyre", description, step 1 (new key/value tokens go into the paged
 *      cache at the slots slot_mapping names).  Slot s names block
 *      s / block_size, offset s % block_size.  Done here one token at a time.
 *
 *  oracle_attention_varlen / oracle_attention_varlen_paged
 *      Steps 4-6 of the same description: a boolean mask of padding validity
 *      plus (for prefill) causality, softmax attention per sequence, output
 *      written only for real tokens.  Grouped-query heads follow the
 *      repeat_interleave expansion of the same description (query head h uses
 *      KV head h / (Hq/Hkv)).  Causality is bottom-right aligned as in
 *      vllm-omni PR #9244 "Support piecewise block-causal attention",
 *      kernel-semantics review: query i of Sq sees key j iff
 *      j <= (Skv - Sq) + i, the attn(Q[s:e], K[:e], causal=True) contract.
 *      A row with no visible key returns zeros, as the CSA2 golden of
 *      TensorRT-LLM PR "CSA2 Vanilla sparse attention" (description: an empty
 *      selection gives zeros).
 *      The _varlen variant takes each sequence's keys/values as plain
 *      logical arrays (geometry from an independent source, as that
 *      TensorRT-LLM description asks of its golden); the _paged variant
 *      reads them through a block table from a cache this file wrote, which
 *      lets a test pin page addressing against the logical form.
 *
 *  oracle_attention_varlen_spans
 *      The piecewise block-causal attention of vllm-omni PR #9244 "Support
 *      piecewise block-causal attention for full_attn_spans" (description:
 *      the shared segment plan).  A sequence's key positions are split into
 *      full segments (the spans, [start, end)) and causal segments (the
 *      rest).  A query at key position p inside a full segment [start, end)
 *      attends bidirectionally to the truncated prefix, keys j < end; any
 *      other query sees keys j <= p, as with plain causal attention.  With
 *      queries and keys aligned this is the description's dense reference,
 *      "key at or before the query, or in the same full block".
 *
 *  oracle_attention_smallseq
 *      ROCm/TransformerEngine PR #461 "CK varlen cross attention for
 *      small-seq", description: one query per batch entry (s_q = 1), keys and
 *      values packed in THD layout with cu_seqlens_kv, no causal mask.
 *
 *  Element types: inputs are bfloat16 bit patterns, or IEEE binary16 (fp16)
 *      bit patterns in the _dtype variants (vllm-spyre PR #853 runs its path
 *      in fp16; ROCm/TransformerEngine PR #461's small-seq path takes BF16
 *      and FP16).  Both widen exactly to double.
 *
 *  oracle_attention_weights
 *      The softmax weights of one (token, head) row, so that a test can check
 *      that they sum to one and that masked keys get none.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* IEEE binary16 (fp16): 1 sign, 5 exponent (bias 15), 10 fraction bits.
   Every value is exact in double: subnormals are f * 2^-24, normals
   (1024 + f) * 2^(e - 25); e == 31 is infinity or NaN. */
static double half_to_double(uint16_t h) {
    int sign = h >> 15, e = (h >> 10) & 0x1f, f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32: widening is exact. */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Cache write                                                               */
/* ------------------------------------------------------------------------ */

/*
 * k, v:             [num_tokens, num_kv_heads, head_dim] bf16 bits
 * slot_mapping:     [num_tokens]; a negative slot means padding: skipped
 * k_cache, v_cache: [num_blocks, block_size, num_kv_heads, head_dim]
 * Returns the number of tokens whose slot lies beyond the pool; those rows are
 * not written.
 */
int64_t oracle_write_kv(const uint16_t *k, const uint16_t *v,
                        const int64_t *slot_mapping, int64_t num_tokens,
                        int num_kv_heads, int head_dim,
                        uint16_t *k_cache, uint16_t *v_cache,
                        int64_t num_blocks, int block_size) {
    int64_t bad = 0;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t block = slot / block_size;
        int64_t offset = slot % block_size;
        if (block >= num_blocks) { ++bad; continue; }
        for (int h = 0; h < num_kv_heads; ++h) {
            for (int d = 0; d < head_dim; ++d) {
                int64_t src = (t * num_kv_heads + h) * (int64_t)head_dim + d;
                int64_t dst = ((block * block_size + offset) * num_kv_heads + h)
                              * (int64_t)head_dim + d;
                k_cache[dst] = k[src];
                v_cache[dst] = v[src];
            }
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------ */
/* Where key j of a sequence lives                                           */
/* ------------------------------------------------------------------------ */

typedef struct {
    /* logical form: rows first_row + j of base, each [num_kv_heads, head_dim] */
    const uint16_t *base;
    int64_t first_row;
    /* paged form (table != NULL): key j sits in block table[j / block_size],
       offset j % block_size of a [num_blocks, block_size, Hkv, D] cache */
    const int32_t *table;
    int block_size;
    int64_t num_blocks;
    int kv_head;
    int num_kv_heads;
    int head_dim;
    double (*widen)(uint16_t);  /* element type: bf16_to_double or half_to_double */
} kv_view;

/* Pointer to the head_dim values of key/value j, or NULL if its block id is
   outside the pool (the caller treats the row as unreadable). */
static const uint16_t *kv_row(const kv_view *c, int64_t j) {
    int64_t row;
    if (c->table) {
        int64_t block = c->table[j / c->block_size];
        if (block < 0 || block >= c->num_blocks) return NULL;
        row = block * c->block_size + j % c->block_size;
    } else {
        row = c->first_row + j;
    }
    return c->base + (row * c->num_kv_heads + c->kv_head) * (int64_t)c->head_dim;
}

/* Number of keys query i (of a sequence with len_q queries and len_kv keys)
   may see: keys 0 .. n-1.  Without causality every key is visible; with it,
   the diagonal is bottom-right aligned. */
static int64_t visible_keys(int64_t i, int64_t len_q, int64_t len_kv, int causal) {
    if (!causal) return len_kv;
    int64_t n = (len_kv - len_q) + i + 1;
    if (n < 0) n = 0;
    if (n > len_kv) n = len_kv;
    return n;
}

/* Keys a query at key position p may see when full segments are given:
   sp[0..2*nsp) holds the sequence's spans as (start, end) pairs.  A span is
   used only if 0 <= start < end <= len_kv and start >= the previous pair's
   end; the others are ignored.  Inside a used span [start, end): keys
   0 .. end-1; otherwise keys 0 .. p (causal).  Returns a count clamped to
   [0, len_kv]. */
static int64_t visible_keys_spans(int64_t p, int64_t len_kv, const int32_t *sp,
                                  int64_t nsp) {
    int64_t n = p + 1;
    int64_t prev_end = 0;
    for (int64_t k = 0; k < nsp; ++k) {
        int64_t a = sp[2 * k], b = sp[2 * k + 1];
        int ok = a >= 0 && a < b && b <= len_kv && a >= prev_end;
        prev_end = b;
        if (ok && p >= a && p < b && b > n) n = b;
    }
    if (n < 0) n = 0;
    if (n > len_kv) n = len_kv;
    return n;
}

/*
 * Score modifiers of one (query token, head) row, auto_round_kernel PR
 * "Migrate CPU SDPA backend" (description: additive masks in the public
 * sdpa(); ALiBi slopes and the TANH30 soft-cap among the kernel library's
 * extensions).  Applied to s_j = scale * <q, k_j> in this order:
 *   soft-cap  s_j <- softcap * tanh(s_j / softcap)          (softcap > 0)
 *   ALiBi     s_j <- s_j + slope * (j - pos)                (has_alibi)
 *   mask      s_j <- s_j + mask_row[j]                      (mask_row)
 * where pos is the query's own key position.  Masking (causal, spans,
 * sequence end) still decides which keys enter the softmax at all.
 */
typedef struct {
    double softcap;
    int has_alibi;
    double slope;
    int64_t pos;
    const float *mask_row;
} row_mods;

/*
 * out[d] = sum_j w_j v_j[d],  w_j = exp(s_j) / sum_i exp(s_i),
 * s_j = scale * <q, k_j> (then the row's modifiers, if any), over keys
 * j < n_vis.  n_vis == 0, or every visible s_j = -inf, gives zeros.
 * The maximum is subtracted inside exp only to keep it finite; it cancels in
 * the ratio.  Returns -1 if some key or value row is unreadable.
 */
static int attention_row(const uint16_t *q, const kv_view *keys,
                         const kv_view *values, int64_t n_vis, int head_dim,
                         double scale, const row_mods *mods, double *out, double *weights,
                         double *s) {
    for (int d = 0; d < head_dim; ++d) out[d] = 0.0;
    if (n_vis <= 0) return 0;
    double m = -INFINITY;
    for (int64_t j = 0; j < n_vis; ++j) {
        const uint16_t *kr = kv_row(keys, j);
        if (!kr) return -1;
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d)
            dot += keys->widen(q[d]) * keys->widen(kr[d]);
        s[j] = scale * dot;
        if (mods) {
            if (mods->softcap > 0.0) s[j] = mods->softcap * tanh(s[j] / mods->softcap);
            if (mods->has_alibi) s[j] += mods->slope * (double)(j - mods->pos);
            if (mods->mask_row) s[j] += (double)mods->mask_row[j];
        }
        if (s[j] > m) m = s[j];
    }
    if (m == -INFINITY) return 0; /* every visible key masked out */
    double denom = 0.0;
    for (int64_t j = 0; j < n_vis; ++j) {
        s[j] = exp(s[j] - m);
        denom += s[j];
    }
    for (int64_t j = 0; j < n_vis; ++j) {
        const uint16_t *vr = kv_row(values, j);
        if (!vr) return -1;
        double w = s[j] / denom;
        if (weights) weights[j] = w;
        for (int d = 0; d < head_dim; ++d) out[d] += w * values->widen(vr[d]);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Variable-length attention (prefill, decode, chunked prefill)              */
/* ------------------------------------------------------------------------ */

/* Score modifiers of a whole call: alibi_slopes [num_q_heads] or NULL; mask
   element (h, t, j) at mask[h * mask_head_stride + t * mask_token_stride + j]
   (t the packed query-token index, j the key position) or NULL. */
typedef struct {
    double softcap;
    const float *alibi_slopes;
    const float *mask;
    int64_t mask_head_stride;
    int64_t mask_token_stride;
} score_mods;

/*
 * Shared driver.  For every requested query token t (all tokens if rows is
 * NULL): find its sequence s, its index i within the sequence, and for every
 * query head h compute attention_row against KV head h / group.
 * Returns 0; -1 for bad head counts; -2 if a block id was outside the pool.
 */
static int varlen_driver(const uint16_t *q, const uint16_t *k_base,
                         const uint16_t *v_base, const int64_t *kv_offsets,
                         const int32_t *block_tables, int max_blocks_per_seq,
                         int block_size, int64_t num_blocks,
                         const int32_t *seq_lens, const int32_t *query_start_loc,
                         int num_seqs, int num_q_heads, int num_kv_heads,
                         int head_dim, double scale, int causal,
                         const int32_t *span_offsets, const int32_t *spans, int dtype,
                         const score_mods *sm,
                         const int64_t *rows, int64_t num_rows, double *out) {
    double (*widen)(uint16_t) = dtype == 1 ? half_to_double : bf16_to_double;
    if (num_kv_heads <= 0 || num_q_heads <= 0 || num_q_heads % num_kv_heads != 0)
        return -1;
    int group = num_q_heads / num_kv_heads;
    int64_t num_q_tokens = query_start_loc[num_seqs];
    int64_t todo = rows ? num_rows : num_q_tokens;
    int64_t max_len = 1;
    for (int s = 0; s < num_seqs; ++s)
        if (seq_lens[s] > max_len) max_len = seq_lens[s];
    int status = 0;

#pragma omp parallel
    {
        double *scratch = (double *)malloc(sizeof(double) * (size_t)max_len);
        /* one task per (query token, query head): rows are independent, and
           so are the heads of a row, so a single decode row still spreads
           over every thread */
#pragma omp for schedule(dynamic, 1)
        for (int64_t task = 0; task < todo * num_q_heads; ++task) {
            int64_t r = task / num_q_heads;
            int h = (int)(task % num_q_heads);
            int64_t t = rows ? rows[r] : r;
            int s = 0;
            while (s < num_seqs && query_start_loc[s + 1] <= t) ++s;
            if (s >= num_seqs) continue;
            int64_t len_q = query_start_loc[s + 1] - query_start_loc[s];
            int64_t len_kv = seq_lens[s];
            int64_t i = t - query_start_loc[s];
            int64_t n_vis = visible_keys(i, len_q, len_kv, causal);
            if (span_offsets) {
                int64_t a = span_offsets[s], b = span_offsets[s + 1];
                n_vis = visible_keys_spans((len_kv - len_q) + i, len_kv,
                                           spans + 2 * a, b > a ? b - a : 0);
            }
            kv_view kview = {0}, vview = {0};
            kview.num_kv_heads = vview.num_kv_heads = num_kv_heads;
            kview.head_dim = vview.head_dim = head_dim;
            kview.kv_head = vview.kv_head = h / group;
            kview.widen = vview.widen = widen;
            kview.base = k_base;
            vview.base = v_base;
            if (block_tables) {
                const int32_t *tab = block_tables + (int64_t)s * max_blocks_per_seq;
                kview.table = vview.table = tab;
                kview.block_size = vview.block_size = block_size;
                kview.num_blocks = vview.num_blocks = num_blocks;
            } else {
                kview.first_row = vview.first_row = kv_offsets[s];
            }
            const uint16_t *qr = q + (t * num_q_heads + h) * (int64_t)head_dim;
            double *o = out + (t * num_q_heads + h) * (int64_t)head_dim;
            row_mods rm, *rmp = NULL;
            if (sm) {
                rm.softcap = sm->softcap;
                rm.has_alibi = sm->alibi_slopes != NULL;
                rm.slope = sm->alibi_slopes ? (double)sm->alibi_slopes[h] : 0.0;
                rm.pos = (len_kv - len_q) + i;
                rm.mask_row = sm->mask ? sm->mask + h * sm->mask_head_stride +
                                             t * sm->mask_token_stride
                                       : NULL;
                rmp = &rm;
            }
            if (attention_row(qr, &kview, &vview, n_vis, head_dim, scale, rmp, o,
                              NULL, scratch) != 0) {
#pragma omp atomic write
                status = -2;
            }
        }
        free(scratch);
    }
    return status;
}

/*
 * Logical form.
 * q:            [num_q_tokens, num_q_heads, head_dim]
 * k_seq, v_seq: sequence s's keys/values are rows kv_offsets[s] ..
 *               kv_offsets[s] + seq_lens[s] - 1, each [num_kv_heads, head_dim]
 * seq_lens:     [num_seqs] key count (prior context + this step's tokens)
 * query_start_loc: [num_seqs + 1] cumulative query offsets
 * rows:         optional query-token indices to compute (NULL = all); other
 *               output rows are left as they are
 * out:          [num_q_tokens, num_q_heads, head_dim] doubles
 */
int oracle_attention_varlen(const uint16_t *q, const uint16_t *k_seq,
                            const uint16_t *v_seq, const int64_t *kv_offsets,
                            const int32_t *seq_lens,
                            const int32_t *query_start_loc, int num_seqs,
                            int num_q_heads, int num_kv_heads, int head_dim,
                            double scale, int causal, const int64_t *rows,
                            int64_t num_rows, double *out) {
    return varlen_driver(q, k_seq, v_seq, kv_offsets, NULL, 0, 1, 0, seq_lens,
                         query_start_loc, num_seqs, num_q_heads, num_kv_heads,
                         head_dim, scale, causal, NULL, NULL, 0, NULL, rows, num_rows, out);
}

/*
 * Logical form with an element type: dtype 0 = bf16, 1 = fp16 (every input
 * is that type's bit pattern); otherwise as oracle_attention_varlen.
 */
int oracle_attention_varlen_dtype(const uint16_t *q, const uint16_t *k_seq,
                                  const uint16_t *v_seq, const int64_t *kv_offsets,
                                  const int32_t *seq_lens,
                                  const int32_t *query_start_loc, int num_seqs,
                                  int num_q_heads, int num_kv_heads, int head_dim,
                                  double scale, int causal, int dtype, const int64_t *rows,
                                  int64_t num_rows, double *out) {
    if (dtype != 0 && dtype != 1) return -1;
    return varlen_driver(q, k_seq, v_seq, kv_offsets, NULL, 0, 1, 0, seq_lens,
                         query_start_loc, num_seqs, num_q_heads, num_kv_heads,
                         head_dim, scale, causal, NULL, NULL, dtype, NULL, rows, num_rows, out);
}

/*
 * Logical form with full segments (see visible_keys_spans): span_offsets
 * [num_seqs + 1] indexes spans [*, 2] int32 (start, end) key positions;
 * sequence s owns pairs span_offsets[s] .. span_offsets[s+1]-1.  Queries
 * outside every full segment are causal.
 */
int oracle_attention_varlen_spans(const uint16_t *q, const uint16_t *k_seq,
                                  const uint16_t *v_seq, const int64_t *kv_offsets,
                                  const int32_t *seq_lens,
                                  const int32_t *query_start_loc, int num_seqs,
                                  int num_q_heads, int num_kv_heads, int head_dim,
                                  double scale, const int32_t *span_offsets,
                                  const int32_t *spans, const int64_t *rows,
                                  int64_t num_rows, double *out) {
    if (!span_offsets || !spans) return -1;
    return varlen_driver(q, k_seq, v_seq, kv_offsets, NULL, 0, 1, 0, seq_lens,
                         query_start_loc, num_seqs, num_q_heads, num_kv_heads,
                         head_dim, scale, 1, span_offsets, spans, 0, NULL, rows, num_rows, out);
}

/*
 * Logical form with score modifiers (see row_mods) and an element type:
 * softcap (0 = off), alibi_slopes [num_q_heads] fp32 or NULL, an additive
 * fp32 mask or NULL with its head / token strides in elements (head stride 0
 * = one mask for every head), and optional full-attention spans as in
 * oracle_attention_varlen_spans (then causal is implied).  Otherwise as
 * oracle_attention_varlen_dtype.
 */
int oracle_attention_varlen_mods(const uint16_t *q, const uint16_t *k_seq,
                                 const uint16_t *v_seq, const int64_t *kv_offsets,
                                 const int32_t *seq_lens,
                                 const int32_t *query_start_loc, int num_seqs,
                                 int num_q_heads, int num_kv_heads, int head_dim,
                                 double scale, int causal, int dtype, double softcap,
                                 const float *alibi_slopes, const float *mask,
                                 int64_t mask_head_stride, int64_t mask_token_stride,
                                 const int32_t *span_offsets, const int32_t *spans,
                                 const int64_t *rows, int64_t num_rows, double *out) {
    if ((dtype != 0 && dtype != 1) || softcap < 0.0) return -1;
    if (span_offsets && !spans) return -1;
    score_mods sm = {softcap, alibi_slopes, mask, mask_head_stride, mask_token_stride};
    return varlen_driver(q, k_seq, v_seq, kv_offsets, NULL, 0, 1, 0, seq_lens,
                         query_start_loc, num_seqs, num_q_heads, num_kv_heads,
                         head_dim, scale, span_offsets ? 1 : causal, span_offsets, spans, dtype,
                         &sm, rows, num_rows, out);
}

/*
 * Paged form: keys/values read through block_tables
 * ([num_seqs, max_blocks_per_seq] int32) from caches shaped
 * [num_blocks, block_size, num_kv_heads, head_dim].
 */
int oracle_attention_varlen_paged(const uint16_t *q, const uint16_t *k_cache,
                                  const uint16_t *v_cache,
                                  const int32_t *block_tables,
                                  int max_blocks_per_seq, const int32_t *seq_lens,
                                  const int32_t *query_start_loc, int num_seqs,
                                  int num_q_heads, int num_kv_heads, int head_dim,
                                  int block_size, int64_t num_blocks,
                                  double scale, int causal, const int64_t *rows,
                                  int64_t num_rows, double *out) {
    return varlen_driver(q, k_cache, v_cache, NULL, block_tables,
                         max_blocks_per_seq, block_size, num_blocks, seq_lens,
                         query_start_loc, num_seqs, num_q_heads, num_kv_heads,
                         head_dim, scale, causal, NULL, NULL, 0, NULL, rows, num_rows, out);
}

/*
 * Softmax weights of query token t, head h (logical form): writes seq_lens[s]
 * doubles, zero for keys the row may not see.  Returns the number of visible
 * keys, or -1 on bad arguments.
 */
int64_t oracle_attention_weights(const uint16_t *q, const uint16_t *k_seq,
                                 const uint16_t *v_seq, const int64_t *kv_offsets,
                                 const int32_t *seq_lens,
                                 const int32_t *query_start_loc, int num_seqs,
                                 int num_q_heads, int num_kv_heads, int head_dim,
                                 double scale, int causal, int64_t t, int h,
                                 double *weights) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return -1;
    int s = 0;
    while (s < num_seqs && query_start_loc[s + 1] <= t) ++s;
    if (s >= num_seqs) return -1;
    int64_t len_q = query_start_loc[s + 1] - query_start_loc[s];
    int64_t len_kv = seq_lens[s];
    int64_t n_vis = visible_keys(t - query_start_loc[s], len_q, len_kv, causal);
    kv_view kview = {0}, vview = {0};
    kview.widen = vview.widen = bf16_to_double;
    kview.base = k_seq;
    vview.base = v_seq;
    kview.first_row = vview.first_row = kv_offsets[s];
    kview.kv_head = vview.kv_head = h / (num_q_heads / num_kv_heads);
    kview.num_kv_heads = vview.num_kv_heads = num_kv_heads;
    kview.head_dim = vview.head_dim = head_dim;
    double *out = (double *)malloc(sizeof(double) * (size_t)head_dim);
    double *scratch = (double *)malloc(sizeof(double) * (size_t)(len_kv > 0 ? len_kv : 1));
    for (int64_t j = 0; j < len_kv; ++j) weights[j] = 0.0;
    const uint16_t *qr = q + (t * num_q_heads + h) * (int64_t)head_dim;
    attention_row(qr, &kview, &vview, n_vis, head_dim, scale, NULL, out, weights, scratch);
    free(out);
    free(scratch);
    return n_vis;
}

/* ------------------------------------------------------------------------ */
/* Small-seq cross attention (s_q = 1, contiguous THD keys/values)           */
/* ------------------------------------------------------------------------ */

/*
 * q:     [batch, num_q_heads, head_dim]       (one query per batch entry)
 * k, v:  [cu_seqlens_kv[batch], num_kv_heads, head_dim]; entry b owns rows
 *        cu_seqlens_kv[b] .. cu_seqlens_kv[b+1] - 1
 * out:   [batch, num_q_heads, head_dim] doubles
 * No causal mask: every key of the entry is visible; an empty entry gives
 * zeros.  Returns 0, or -1 on bad head counts.
 */
static int smallseq_driver(const uint16_t *q, const uint16_t *k,
                           const uint16_t *v, const int32_t *cu_seqlens_kv,
                           int batch, int num_q_heads, int num_kv_heads,
                           int head_dim, double scale, int dtype, double *out) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return -1;
    double (*widen)(uint16_t) = dtype == 1 ? half_to_double : bf16_to_double;
    int group = num_q_heads / num_kv_heads;
    int64_t max_len = 1;
    for (int b = 0; b < batch; ++b) {
        int64_t n = (int64_t)cu_seqlens_kv[b + 1] - cu_seqlens_kv[b];
        if (n > max_len) max_len = n;
    }
#pragma omp parallel
    {
        double *scratch = (double *)malloc(sizeof(double) * (size_t)max_len);
#pragma omp for schedule(static)
        for (int b = 0; b < batch; ++b) {
            int64_t n = (int64_t)cu_seqlens_kv[b + 1] - cu_seqlens_kv[b];
            for (int h = 0; h < num_q_heads; ++h) {
                kv_view kview = {0}, vview = {0};
                kview.base = k;
                vview.base = v;
                kview.first_row = vview.first_row = cu_seqlens_kv[b];
                kview.kv_head = vview.kv_head = h / group;
                kview.num_kv_heads = vview.num_kv_heads = num_kv_heads;
                kview.head_dim = vview.head_dim = head_dim;
                kview.widen = vview.widen = widen;
                const uint16_t *qr = q + ((int64_t)b * num_q_heads + h) * head_dim;
                double *o = out + ((int64_t)b * num_q_heads + h) * head_dim;
                attention_row(qr, &kview, &vview, n, head_dim, scale, NULL, o, NULL,
                              scratch);
            }
        }
        free(scratch);
    }
    return 0;
}

int oracle_attention_smallseq(const uint16_t *q, const uint16_t *k,
                              const uint16_t *v, const int32_t *cu_seqlens_kv,
                              int batch, int num_q_heads, int num_kv_heads,
                              int head_dim, double scale, double *out) {
    return smallseq_driver(q, k, v, cu_seqlens_kv, batch, num_q_heads, num_kv_heads,
                           head_dim, scale, 0, out);
}

/* The same with an element type: dtype 0 = bf16, 1 = fp16. */
int oracle_attention_smallseq_dtype(const uint16_t *q, const uint16_t *k,
                                    const uint16_t *v, const int32_t *cu_seqlens_kv,
                                    int batch, int num_q_heads, int num_kv_heads,
                                    int head_dim, double scale, int dtype, double *out) {
    if (dtype != 0 && dtype != 1) return -1;
    return smallseq_driver(q, k, v, cu_seqlens_kv, batch, num_q_heads, num_kv_heads,
                           head_dim, scale, dtype, out);
}

/*
 * Small-seq attention weights and backward (ROCm/TransformerEngine PR #461,
 * description: the forward also returns the attention weights, shaped
 * [batch, Hq, 1, max_seqlen_kv]; the backward computes grad_V, grad_attn,
 * the softmax backward and grad_Q / grad_K).  With s_j = scale * <q, k_j>,
 * p = softmax(s) over the entry's keys and upstream gradient dO:
 *     dV_j += p_j dO                    (summed over the query heads sharing
 *     dP_j  = <dO, v_j>                  a KV head)
 *     dS_j  = p_j (dP_j - sum_k p_k dP_k)
 *     dQ    = scale * sum_j dS_j k_j
 *     dK_j += scale * dS_j q
 * weights: [batch, Hq, wlen] doubles (entry b's p in the first n_b slots,
 * zeros after); dq [batch, Hq, D]; dk, dv [total keys, Hkv, D] doubles.
 * The backward takes p either recomputed from q and k (weights NULL) or as
 * given (the weights the forward saved, which is what the PR's backward
 * reads); the formulas above are the same either way.
 * An empty entry has no weights and contributes nothing.
 */
/* p_j = softmax_j(scale * <q, k_j>) over the n keys of one entry and KV head. */
static void smallseq_probs(const uint16_t *q, const uint16_t *k, int64_t first, int64_t n,
                           int kvh, int num_kv_heads, int head_dim, double scale,
                           double (*widen)(uint16_t), double *p) {
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        const uint16_t *kr = k + ((first + j) * num_kv_heads + kvh) * (int64_t)head_dim;
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d) dot += widen(q[d]) * widen(kr[d]);
        p[j] = scale * dot;
        if (p[j] > m) m = p[j];
    }
    double denom = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        p[j] = exp(p[j] - m);
        denom += p[j];
    }
    for (int64_t j = 0; j < n; ++j) p[j] /= denom;
}

int oracle_smallseq_weights(const uint16_t *q, const uint16_t *k,
                            const int32_t *cu_seqlens_kv, int batch, int num_q_heads,
                            int num_kv_heads, int head_dim, double scale, int dtype,
                            int wlen, double *weights) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || wlen < 0) return -1;
    double (*widen)(uint16_t) = dtype == 1 ? half_to_double : bf16_to_double;
    int group = num_q_heads / num_kv_heads;
    for (int b = 0; b < batch; ++b) {
        int64_t first = cu_seqlens_kv[b], n = (int64_t)cu_seqlens_kv[b + 1] - first;
        if (n > wlen) return -2;
        for (int h = 0; h < num_q_heads; ++h) {
            double *w = weights + ((int64_t)b * num_q_heads + h) * wlen;
            for (int j = 0; j < wlen; ++j) w[j] = 0.0;
            if (n <= 0) continue;
            smallseq_probs(q + ((int64_t)b * num_q_heads + h) * head_dim, k, first, n,
                           h / group, num_kv_heads, head_dim, scale, widen, w);
        }
    }
    return 0;
}

int oracle_smallseq_backward(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                             const uint16_t *dout, const int32_t *cu_seqlens_kv, int batch,
                             int num_q_heads, int num_kv_heads, int head_dim, double scale,
                             int dtype, const double *weights, int wlen, double *dq,
                             double *dk, double *dv) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return -1;
    if (weights && wlen <= 0) return -1;
    double (*widen)(uint16_t) = dtype == 1 ? half_to_double : bf16_to_double;
    int group = num_q_heads / num_kv_heads;
    int64_t total = cu_seqlens_kv[batch];
    for (int64_t i = 0; i < total * num_kv_heads * head_dim; ++i) dk[i] = dv[i] = 0.0;
    for (int64_t i = 0; i < (int64_t)batch * num_q_heads * head_dim; ++i) dq[i] = 0.0;
    int64_t max_len = 1;
    for (int b = 0; b < batch; ++b) {
        int64_t n = (int64_t)cu_seqlens_kv[b + 1] - cu_seqlens_kv[b];
        if (n > max_len) max_len = n;
    }
    double *p = (double *)malloc(sizeof(double) * (size_t)max_len);
    double *dp = (double *)malloc(sizeof(double) * (size_t)max_len);
    for (int b = 0; b < batch; ++b) {
        int64_t first = cu_seqlens_kv[b], n = (int64_t)cu_seqlens_kv[b + 1] - first;
        if (n <= 0) continue;
        for (int h = 0; h < num_q_heads; ++h) {
            int kvh = h / group;
            const uint16_t *qr = q + ((int64_t)b * num_q_heads + h) * head_dim;
            const uint16_t *gr = dout + ((int64_t)b * num_q_heads + h) * head_dim;
            if (weights) { /* the forward's saved weights, as the backward reads them */
                if (n > wlen) { free(p); free(dp); return -2; }
                const double *w = weights + ((int64_t)b * num_q_heads + h) * wlen;
                for (int64_t j = 0; j < n; ++j) p[j] = w[j];
            } else {
                smallseq_probs(qr, k, first, n, kvh, num_kv_heads, head_dim, scale, widen, p);
            }
            double sum_pdp = 0.0;
            for (int64_t j = 0; j < n; ++j) {
                const uint16_t *vr = v + ((first + j) * num_kv_heads + kvh) * (int64_t)head_dim;
                double dot = 0.0;
                for (int d = 0; d < head_dim; ++d) dot += widen(gr[d]) * widen(vr[d]);
                dp[j] = dot;
                sum_pdp += p[j] * dot;
            }
            double *dqr = dq + ((int64_t)b * num_q_heads + h) * head_dim;
            for (int64_t j = 0; j < n; ++j) {
                double ds = p[j] * (dp[j] - sum_pdp);
                const uint16_t *kr = k + ((first + j) * num_kv_heads + kvh) * (int64_t)head_dim;
                double *dkr = dk + ((first + j) * num_kv_heads + kvh) * (int64_t)head_dim;
                double *dvr = dv + ((first + j) * num_kv_heads + kvh) * (int64_t)head_dim;
                for (int d = 0; d < head_dim; ++d) {
                    dqr[d] += scale * ds * widen(kr[d]);
                    dkr[d] += scale * ds * widen(qr[d]);
                    dvr[d] += p[j] * widen(gr[d]);
                }
            }
        }
    }
    free(p);
    free(dp);
    return 0;
}

/* One element widened exactly (dtype 0 = bf16, 1 = fp16), for tests. */
double oracle_widen(uint16_t bits, int dtype) {
    return dtype == 1 ? half_to_double(bits) : bf16_to_double(bits);
}
