/*
 * oracle.c -- plain, slow, obviously correct CPU oracle for the paged KV-cache
 * hot path (PagedAttention decode, KV append, copy-on-write block copy).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library may include, link
 * or call this file.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference leg use it.  It shares no code with the CUDA path.
 *
 * Sources (pages, by title and section):
 *  - "PagedAttention" glossary entry (ultralytics.com/es/glossary/pagedattention),
 *    section "Como funciona la paginacion": the cache is split into blocks of a
 *    fixed number of tokens (16 by default), a block table records their order,
 *    and the attention kernel gathers keys and values block by block through it.
 *    Its worked PyTorch example addresses token `pos` at
 *    (block_table[pos // block_size], pos % block_size) of a shared pool indexed
 *    [block, slot, dim] and reads a request back with
 *    pool[block_table].reshape(-1, head_dim)[:len].
 *  - same page, section "Compartir bloques entre secuencias": blocks are shared
 *    through tables with a per-block reference count; a writer copies a block
 *    other sequences still use before writing it (copy-on-write).
 *  - same page, section "Tecnicas relacionadas": grouped-query attention shares
 *    key/value heads among query heads; FP8 KV cache stores 8-bit values.
 *  - "Le cache KV et PagedAttention" (gyaansetu.com/fr/ai/-1d481f), section
 *    "Qu'est-ce que le KV Cache ?": token n+1 attends to the K and V of tokens
 *    1..n; each step appends only the new token's K and V to the cache.
 *  - The attention formula softmax(q K^T * scale) V is not written on the pages;
 *    it is the standard definition of (single-query) scaled dot-product attention.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - pool layout [num_blocks][block_size][num_kv_heads][head_dim], separate K
 *    and V pools (the glossary example's [block, slot, dim] with heads appended);
 *  - query head h uses key/value head h / (num_heads / num_kv_heads);
 *  - context length 0 produces a zero output;
 *  - a slot < 0 in a write is padding and is skipped; a slot or block id out
 *    of range is skipped and counted;
 *  - FP8 is OCP OFP8 E4M3 (bias 7, max finite 448, no infinities, NaN = S.1111.111);
 *    a write divides in IEEE fp32 (x / scale) and encodes with round to nearest,
 *    ties to even, saturating to +-448; a read multiplies the decoded value by
 *    the per-tensor scale.
 *
 * All attention arithmetic is in double precision.  Every input element is
 * converted exactly to double (bf16 and fp32 embed exactly; every E4M3 code
 * decodes exactly).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_FP8_E4M3 = 2 };

static size_t elem_size(int dtype) {
    return dtype == ORC_F32 ? 4 : dtype == ORC_BF16 ? 2 : 1;
}

/* ---------------------------------------------------------------- formats */

/* bf16 is the top half of an IEEE binary32; widening is exact. */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static float bf16_to_float(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* OCP OFP8 E4M3, from the format definition: 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits.  Exponent field 0 encodes subnormals m/8 * 2^-6.
 * S.1111.111 is NaN; there are no infinities, so S.1111.110 = 448 is the
 * largest finite magnitude. */
double orc_e4m3_decode(uint8_t code) {
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* Encode a binary32 value to E4M3: round to nearest, ties to even, saturate
 * finite overflow (and infinities) to the largest finite magnitude 448.
 * NaN encodes to 0x7F.  The search walks the 127 non-negative finite codes,
 * which are ordered by magnitude, and picks between the two neighbours of |x|
 * by comparing |x| with their exact midpoint (all values are exact in double). */
uint8_t orc_e4m3_encode(float x) {
    uint8_t sign;
    double a;
    int c;
    if (isnan(x)) return 0x7F;
    sign = signbit(x) ? 0x80 : 0x00;
    a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    /* largest code c with decode(c) <= a; codes 0x00..0x7E ascend */
    c = 0;
    while (c < 0x7E && orc_e4m3_decode((uint8_t)(c + 1)) <= a) c++;
    if (orc_e4m3_decode((uint8_t)c) != a) {
        double lo = orc_e4m3_decode((uint8_t)c);
        double hi = orc_e4m3_decode((uint8_t)(c + 1));
        double mid = (lo + hi) / 2.0;
        if (a > mid || (a == mid && (c & 1))) c = c + 1;
    }
    return (uint8_t)(sign | c);
}

/* Quantise one bf16 or fp32 source element for an FP8 cache: IEEE fp32
 * division by the per-tensor scale, then the encoder above. */
static uint8_t quantise(float x, float scale) {
    float q = x / scale;
    return orc_e4m3_encode(q);
}

static double load_elem(const void* base, int dtype, size_t idx) {
    if (dtype == ORC_F32) {
        float f;
        memcpy(&f, (const char*)base + 4 * idx, 4);
        return (double)f;
    }
    if (dtype == ORC_BF16) {
        uint16_t b;
        memcpy(&b, (const char*)base + 2 * idx, 2);
        return bf16_to_double(b);
    }
    return orc_e4m3_decode(((const uint8_t*)base)[idx]);
}

static float load_src_float(const void* base, int dtype, size_t idx) {
    if (dtype == ORC_F32) {
        float f;
        memcpy(&f, (const char*)base + 4 * idx, 4);
        return f;
    }
    {
        uint16_t b;
        memcpy(&b, (const char*)base + 2 * idx, 2);
        return bf16_to_float(b);
    }
}

/* ---------------------------------------------------------------- KV write */

/* KV append (the "reshape and cache" step): token i's K and V, laid out
 * [num_tokens][num_kv_heads][head_dim], go to slot slot_mapping[i] of the pools,
 * where slot = block * block_size + offset addresses row (block, offset) of the
 * [num_blocks][block_size][num_kv_heads][head_dim] pool.  Same-dtype writes are
 * byte copies; an FP8 cache stores quantise(x, scale).  Returns the number of
 * out-of-range slots skipped. */
int orc_kv_write(const void* k, const void* v, int src_dtype, const int64_t* slot_mapping,
                 int num_tokens, void* k_pool, void* v_pool, int cache_dtype, int num_blocks,
                 int block_size, int num_kv_heads, int head_dim, float k_scale, float v_scale) {
    size_t row = (size_t)num_kv_heads * (size_t)head_dim;
    int bad = 0;
    int i;
    for (i = 0; i < num_tokens; i++) {
        int64_t slot = slot_mapping[i];
        size_t e;
        if (slot < 0) continue;
        if (slot >= (int64_t)num_blocks * block_size) {
            bad++;
            continue;
        }
        if (cache_dtype == src_dtype) {
            size_t es = elem_size(src_dtype);
            memcpy((char*)k_pool + (size_t)slot * row * es, (const char*)k + (size_t)i * row * es, row * es);
            memcpy((char*)v_pool + (size_t)slot * row * es, (const char*)v + (size_t)i * row * es, row * es);
        } else if (cache_dtype == ORC_FP8_E4M3) {
            for (e = 0; e < row; e++) {
                ((uint8_t*)k_pool)[(size_t)slot * row + e] =
                    quantise(load_src_float(k, src_dtype, (size_t)i * row + e), k_scale);
                ((uint8_t*)v_pool)[(size_t)slot * row + e] =
                    quantise(load_src_float(v, src_dtype, (size_t)i * row + e), v_scale);
            }
        } else {
            return -1; /* unsupported combination */
        }
    }
    return bad;
}

/* ---------------------------------------------------------------- block copy */

/* Copy-on-write block copy: for every (src, dst) pair copy the whole physical
 * block (all slots, all heads) in both pools.  Pairs whose ids fall outside
 * [0, num_blocks) are skipped and counted.  A dst that repeats, or that is also
 * some pair's src, makes the result order-dependent; the oracle refuses such a
 * list (returns -1) instead of picking an order. */
int orc_copy_blocks(void* k_pool, void* v_pool, size_t block_bytes, const int64_t* pairs,
                    int num_pairs, int num_blocks) {
    int i, j, bad = 0;
    for (i = 0; i < num_pairs; i++) {
        for (j = 0; j < num_pairs; j++) {
            if (i != j && pairs[2 * i + 1] == pairs[2 * j + 1]) return -1;
            if (pairs[2 * i + 1] == pairs[2 * j]) return -1;
        }
    }
    for (i = 0; i < num_pairs; i++) {
        int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
        if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) {
            bad++;
            continue;
        }
        memcpy((char*)k_pool + (size_t)d * block_bytes, (const char*)k_pool + (size_t)s * block_bytes, block_bytes);
        memcpy((char*)v_pool + (size_t)d * block_bytes, (const char*)v_pool + (size_t)s * block_bytes, block_bytes);
    }
    return bad;
}

/* Swap between pools (fine-grained eviction: pages move to host memory and
 * back, "Le cache KV et PagedAttention", gyaansetu.com): for every (src, dst)
 * pair copy block src of the source pools over block dst of the destination
 * pools.  The pools are distinct, so only a repeated dst is order-dependent
 * (refused: -1).  Pairs outside their pool's range are skipped and counted. */
int orc_swap_blocks(void* dst_k, void* dst_v, int dst_blocks, const void* src_k, const void* src_v,
                    int src_blocks, size_t block_bytes, const int64_t* pairs, int num_pairs) {
    int i, j, bad = 0;
    for (i = 0; i < num_pairs; i++)
        for (j = i + 1; j < num_pairs; j++)
            if (pairs[2 * i + 1] == pairs[2 * j + 1]) return -1;
    for (i = 0; i < num_pairs; i++) {
        int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
        if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) {
            bad++;
            continue;
        }
        memcpy((char*)dst_k + (size_t)d * block_bytes, (const char*)src_k + (size_t)s * block_bytes, block_bytes);
        memcpy((char*)dst_v + (size_t)d * block_bytes, (const char*)src_v + (size_t)s * block_bytes, block_bytes);
    }
    return bad;
}

/* ---------------------------------------------------------------- gather */

/* The worked example's read-back: the bytes of a request's first `len` tokens
 * in logical order, taken through its block table from a pool of rows of
 * `row_bytes` (one row = one slot of one block).  out receives len*row_bytes.
 * Returns the number of table entries outside [0, num_blocks) (rows left 0). */
int orc_gather(const void* pool, size_t row_bytes, const int32_t* table, int len, int block_size,
               int num_blocks, void* out) {
    int t, bad = 0;
    for (t = 0; t < len; t++) {
        int32_t blk = table[t / block_size];
        if (blk < 0 || blk >= num_blocks) {
            memset((char*)out + (size_t)t * row_bytes, 0, row_bytes);
            bad++;
            continue;
        }
        memcpy((char*)out + (size_t)t * row_bytes,
               (const char*)pool + ((size_t)blk * block_size + (size_t)(t % block_size)) * row_bytes, row_bytes);
    }
    return bad;
}

/* ---------------------------------------------------------------- attention */

/* Logical token t of sequence s, key/value head g: element offset of its row. */
static int token_row(const int32_t* table, int t, int block_size, int num_blocks, int num_kv_heads, int g,
                     int head_dim, size_t* off) {
    int32_t blk = table[t / block_size];
    if (blk < 0 || blk >= num_blocks) return 0;
    *off = (((size_t)blk * block_size + (size_t)(t % block_size)) * num_kv_heads + g) * head_dim;
    return 1;
}

/* Attention of one query head over logical tokens [t0, t1) of one sequence:
 * scores s_t = scale * sum_d q[d] * K[t][d]; m = max s_t; l = sum exp(s_t - m);
 * o = sum exp(s_t - m) V[t] / l.  Tokens whose block id is out of range are
 * left out.  Returns the number of tokens used. */
static int attend_range(const double* qv, const void* k_pool, const void* v_pool, int cache_dtype,
                        const int32_t* table, int t0, int t1, int block_size, int num_blocks,
                        int num_kv_heads, int g, int head_dim, double scale, double k_scale,
                        double v_scale, double* scores, double* m_out, double* l_out, double* o) {
    int t, d, used = 0;
    double m = -INFINITY, l = 0.0;
    size_t off;
    for (d = 0; d < head_dim; d++) o[d] = 0.0;
    for (t = t0; t < t1; t++) {
        double dot = 0.0;
        if (!token_row(table, t, block_size, num_blocks, num_kv_heads, g, head_dim, &off)) {
            scores[t - t0] = -INFINITY;
            continue;
        }
        for (d = 0; d < head_dim; d++) dot += qv[d] * (load_elem(k_pool, cache_dtype, off + d) * k_scale);
        scores[t - t0] = scale * dot;
        if (scores[t - t0] > m) m = scores[t - t0];
        used++;
    }
    if (used == 0) {
        *m_out = -INFINITY;
        *l_out = 0.0;
        return 0;
    }
    for (t = t0; t < t1; t++) {
        double w;
        if (scores[t - t0] == -INFINITY) continue;
        w = exp(scores[t - t0] - m);
        l += w;
        token_row(table, t, block_size, num_blocks, num_kv_heads, g, head_dim, &off);
        for (d = 0; d < head_dim; d++) o[d] += w * (load_elem(v_pool, cache_dtype, off + d) * v_scale);
    }
    for (d = 0; d < head_dim; d++) o[d] /= l;
    *m_out = m;
    *l_out = l;
    return used;
}

/* Single-query decode attention through block tables.
 *   out  [num_seqs][num_heads][head_dim] (double)
 *   q    [num_seqs][num_heads][head_dim] in q_dtype (fp32 or bf16)
 *   pools [num_blocks][block_size][num_kv_heads][head_dim] in cache_dtype
 *   block_tables [num_seqs][max_blocks_per_seq], context_lens [num_seqs]
 * partition_tokens <= 0: one pass over the whole context.  Otherwise the context
 * is cut into partitions of partition_tokens tokens; each yields (m_p, l_p, o_p)
 * and the partitions are merged: M = max m_p, w_p = l_p exp(m_p - M),
 * out = sum_p w_p o_p / sum_p w_p.
 * Returns the number of referenced table entries (per sequence, tokens < len)
 * that were out of range, or -1 for bad arguments. */
int orc_paged_attention_decode(double* out, const void* q, int q_dtype, const void* k_pool,
                               const void* v_pool, int cache_dtype, const int32_t* block_tables,
                               int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                               int num_blocks, int block_size, int num_heads, int num_kv_heads,
                               int head_dim, double scale, double k_scale, double v_scale,
                               int partition_tokens, int num_threads) {
    int bad = 0, s, pair;
    int group;
    if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || head_dim <= 0 ||
        block_size <= 0)
        return -1;
    group = num_heads / num_kv_heads;
    for (s = 0; s < num_seqs; s++) {
        int L = context_lens[s], j;
        if (L > max_blocks_per_seq * block_size) return -1;
        for (j = 0; j < (L + block_size - 1) / block_size; j++) {
            int32_t b = block_tables[(size_t)s * max_blocks_per_seq + j];
            if (b < 0 || b >= num_blocks) bad++;
        }
    }
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (pair = 0; pair < num_seqs * num_heads; pair++) {
        int s2 = pair / num_heads, h = pair % num_heads;
        int g = h / group;
        int L = context_lens[s2];
        const int32_t* table = block_tables + (size_t)s2 * max_blocks_per_seq;
        double* o = out + ((size_t)s2 * num_heads + h) * head_dim;
        double* qv = (double*)malloc(sizeof(double) * head_dim);
        double* acc = (double*)malloc(sizeof(double) * head_dim);
        double* part_o = (double*)malloc(sizeof(double) * head_dim);
        double* scores;
        int d;
        for (d = 0; d < head_dim; d++) qv[d] = load_elem(q, q_dtype, ((size_t)s2 * num_heads + h) * head_dim + d);
        if (L <= 0) {
            for (d = 0; d < head_dim; d++) o[d] = 0.0;
        } else if (partition_tokens <= 0) {
            double m, l;
            scores = (double*)malloc(sizeof(double) * L);
            if (attend_range(qv, k_pool, v_pool, cache_dtype, table, 0, L, block_size, num_blocks,
                             num_kv_heads, g, head_dim, scale, k_scale, v_scale, scores, &m, &l, part_o) == 0)
                for (d = 0; d < head_dim; d++) o[d] = 0.0;
            else
                for (d = 0; d < head_dim; d++) o[d] = part_o[d];
            free(scores);
        } else {
            int nparts = (L + partition_tokens - 1) / partition_tokens, p;
            double* pm = (double*)malloc(sizeof(double) * nparts);
            double* pl = (double*)malloc(sizeof(double) * nparts);
            double* po = (double*)malloc(sizeof(double) * (size_t)nparts * head_dim);
            double M = -INFINITY, W = 0.0;
            scores = (double*)malloc(sizeof(double) * partition_tokens);
            for (p = 0; p < nparts; p++) {
                int t0 = p * partition_tokens;
                int t1 = t0 + partition_tokens < L ? t0 + partition_tokens : L;
                attend_range(qv, k_pool, v_pool, cache_dtype, table, t0, t1, block_size, num_blocks,
                             num_kv_heads, g, head_dim, scale, k_scale, v_scale, scores, &pm[p], &pl[p],
                             po + (size_t)p * head_dim);
                if (pm[p] > M) M = pm[p];
            }
            for (d = 0; d < head_dim; d++) acc[d] = 0.0;
            if (M != -INFINITY) {
                for (p = 0; p < nparts; p++) {
                    double w;
                    if (pl[p] == 0.0) continue;
                    w = pl[p] * exp(pm[p] - M);
                    W += w;
                    for (d = 0; d < head_dim; d++) acc[d] += w * po[(size_t)p * head_dim + d];
                }
            }
            for (d = 0; d < head_dim; d++) o[d] = W > 0.0 ? acc[d] / W : 0.0;
            free(pm);
            free(pl);
            free(po);
            free(scores);
        }
        free(qv);
        free(acc);
        free(part_o);
    }
    return bad;
}

/* Causal multi-token attention through block tables (the prompt pass: the
 * prompt's blocks are allocated first and then filled, and attention reads
 * them through the table in logical order, iplexlaw.co.kr, section on logical
 * vs physical order; every token attends to all the tokens before it,
 * gyaansetu.com, KV-cache definition).
 * Sequence s has nq = query_start[s+1] - query_start[s] new tokens: the last
 * nq of its context_lens[s] tokens, whose K/V are already in the pools.  Query
 * row r = query_start[s] + i is at position p = context_lens[s] - nq + i and
 * attends to tokens t <= p, exactly as a single-query decode over p + 1
 * tokens would.
 *   out [total_q][num_heads][head_dim] (double); q [total_q][num_heads][head_dim]
 *   row_mask: NULL, or uint8 [total_q]: rows with 0 are skipped (left 0)
 * Returns the number of out-of-range table entries among each sequence's
 * first context_lens[s] tokens, or -1 for bad arguments (nq > context). */
int orc_paged_attention_prefill(double* out, const void* q, int q_dtype, const void* k_pool,
                                const void* v_pool, int cache_dtype, const int32_t* block_tables,
                                int max_blocks_per_seq, const int32_t* context_lens,
                                const int32_t* query_start, int num_seqs, int num_blocks, int block_size,
                                int num_heads, int num_kv_heads, int head_dim, double scale,
                                double k_scale, double v_scale, const uint8_t* row_mask, int num_threads) {
    int bad = 0, s, group, total;
    long long pair;
    if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || head_dim <= 0 ||
        block_size <= 0 || num_seqs < 0 || query_start[0] != 0)
        return -1;
    group = num_heads / num_kv_heads;
    for (s = 0; s < num_seqs; s++) {
        int L = context_lens[s], nq = query_start[s + 1] - query_start[s], j;
        if (nq < 0 || nq > L || L > max_blocks_per_seq * block_size) return -1;
        for (j = 0; j < (L + block_size - 1) / block_size; j++) {
            int32_t b = block_tables[(size_t)s * max_blocks_per_seq + j];
            if (b < 0 || b >= num_blocks) bad++;
        }
    }
    total = query_start[num_seqs];
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (pair = 0; pair < (long long)total * num_heads; pair++) {
        int r = (int)(pair / num_heads), h = (int)(pair % num_heads);
        int s2 = 0, d, pos;
        double m, l;
        double* o = out + ((size_t)r * num_heads + h) * head_dim;
        double* qv;
        double* scores;
        if (row_mask != NULL && !row_mask[r]) continue;
        while (query_start[s2 + 1] <= r) s2++;  /* the sequence holding row r */
        pos = context_lens[s2] - (query_start[s2 + 1] - query_start[s2]) + (r - query_start[s2]);
        qv = (double*)malloc(sizeof(double) * head_dim);
        scores = (double*)malloc(sizeof(double) * (pos + 1));
        for (d = 0; d < head_dim; d++) qv[d] = load_elem(q, q_dtype, ((size_t)r * num_heads + h) * head_dim + d);
        if (attend_range(qv, k_pool, v_pool, cache_dtype, block_tables + (size_t)s2 * max_blocks_per_seq, 0,
                         pos + 1, block_size, num_blocks, num_kv_heads, h / group, head_dim, scale, k_scale,
                         v_scale, scores, &m, &l, o) == 0)
            for (d = 0; d < head_dim; d++) o[d] = 0.0;
        free(qv);
        free(scores);
    }
    return bad;
}

/* Size in bytes of a KV cache: 2 (K and V) * layers * kv heads * head_dim *
 * element bytes per token, times the number of tokens. */
double orc_kv_cache_bytes(int layers, int num_kv_heads, int head_dim, int elem_bytes, double tokens) {
    return 2.0 * layers * num_kv_heads * head_dim * elem_bytes * tokens;
}

int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
