/*
 * pkv_oracle.c -- plain, slow, fp64 CPU oracle for the paged KV cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the test suite, the smoke check and the CPU-baseline /
 * reference leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA library; the two meet only in the seeded input
 * generators, which hold none of the method's arithmetic.
 *
 * Sources (web pages about vLLM; they print no code for the kernel itself):
 *   [YK]  "大模型推理框架 vLLM 源码解析 一" (ai.yueke.cloud), section 三
 *         "vLLM 源码关键路径解析": key_cache / value_cache have the shape
 *         [num_blocks, block_size, num_heads, head_dim]; decode walks
 *         j = 0 .. context_lens[i]-1, takes the physical block
 *         block_tables[i][j // block_size] and the in-block offset
 *         j % block_size, and reads the key there ("zero-copy access"); the
 *         score / softmax step is left as a comment on that page.
 *   [FC]  "23.1 vLLM：高吞吐推理框架原理与部署" (r.flycode100.com), section 二
 *         "PagedAttention 的核心原理", part 2: blocks of 16 tokens, a block
 *         table keeps the logical order, blocks need not be physically
 *         contiguous; the kernel locates the scattered blocks through the
 *         table and computes attention piece by piece.
 *   [MH]  "大模型推理框架VLLM-0.7.3源码" (mhpq.cn), sections 2.1 and 3.3:
 *         the model runner produces slot_mapping, telling the operator into
 *         which cell each current token's K/V is written.
 *
 * Readings where the pages are silent (each is the plainest one the rest
 * supports):
 *   - scores are scale * <q, k>, followed by the standard softmax over the
 *     sequence's first context_len tokens and a weighted sum of V (the step
 *     the [YK] pseudocode elides);
 *   - grouped-query attention: query head h reads kv head h / (Hq / Hkv);
 *   - slot = physical_block * block_size + offset; a negative slot marks a
 *     padding token and is skipped;
 *   - context_len == 0 gives an all-zero output;
 *   - split-context decode: partition p covers logical tokens
 *     [p*P, min(L, (p+1)*P)); its (max, sum of exp, normalised output) are
 *     merged by weighting each with exp(m_p - M) * l_p.
 *
 * Element types are 16-bit storage codes: dtype 0 = IEEE binary16 (fp16),
 * dtype 1 = bfloat16.  Both are decoded to double exactly, from their bit
 * fields, below.  All arithmetic is double precision, in the order the
 * definitions state it; no blocking, fusion or reordering.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define PKVO_OK 0
#define PKVO_ERR_ARG 1
#define PKVO_ERR_RANGE 3

/* ---- element decoding ------------------------------------------------- */

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double pkvo_decode_f16(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);               /* zero / subnormal: f * 2^-24 */
    else if (e == 31)
        v = (f == 0) ? INFINITY : NAN;
    else
        v = ldexp((double)(1024 + f), e - 25);   /* (1 + f/2^10) * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double pkvo_decode_bf16(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int e = (b >> 7) & 0xff;
    int f = b & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133);              /* zero / subnormal: f * 2^-133 */
    else if (e == 255)
        v = (f == 0) ? INFINITY : NAN;
    else
        v = ldexp((double)(128 + f), e - 134);   /* (1 + f/2^7) * 2^(e-127) */
    return sign ? -v : v;
}

static double decode(uint16_t x, int dtype)
{
    return dtype == 0 ? pkvo_decode_f16(x) : pkvo_decode_bf16(x);
}

void pkvo_decode_array(const uint16_t *src, int64_t n, int dtype, double *dst)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = decode(src[i], dtype);
}

/* ---- KV write through slot_mapping ([MH] 2.1, 3.3) ---------------------- */

/*
 * For every new token t and kv head h:
 *   key_cache[slot / bs, slot % bs, h, :] = key[t, h, :]   (bit copy)
 *   value_cache[...]                      = value[t, h, :]
 * with slot = slot_mapping[t].  Negative slots are padding and skipped.  A
 * slot >= num_blocks * block_size is an error: nothing is written for any
 * token and PKVO_ERR_RANGE is returned.
 */
int pkvo_kv_cache_write(const uint16_t *key, const uint16_t *value,
                        const int64_t *slot_mapping, int64_t num_tokens,
                        int num_kv_heads, int head_dim,
                        uint16_t *key_cache, uint16_t *value_cache,
                        int64_t num_blocks, int block_size)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
        return PKVO_ERR_ARG;
    for (int64_t t = 0; t < num_tokens; ++t)
        if (slot_mapping[t] >= num_blocks * (int64_t)block_size)
            return PKVO_ERR_RANGE;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        int64_t block = slot / block_size;
        int64_t offset = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * (int64_t)head_dim;
            int64_t src = (t * num_kv_heads + h) * (int64_t)head_dim;
            for (int d = 0; d < head_dim; ++d) {
                key_cache[dst + d] = key[src + d];
                value_cache[dst + d] = value[src + d];
            }
        }
    }
    return PKVO_OK;
}

/* ---- block copy: copy-on-write and swap ([FC] 二.3; [YK] 三 swap to CPU) -- */

/*
 * For every pair i: the whole block src_cache[mapping[2i]] (block_elems
 * 16-bit elements) is copied bit for bit to dst_cache[mapping[2i+1]].  A
 * block id outside its pool is an error: nothing is copied and
 * PKVO_ERR_RANGE is returned.  Pairs are applied in order.
 */
int pkvo_copy_blocks(const uint16_t *src_cache, uint16_t *dst_cache, const int32_t *mapping,
                     int num_pairs, int64_t src_blocks, int64_t dst_blocks, int64_t block_elems)
{
    if (num_pairs < 0 || block_elems <= 0)
        return PKVO_ERR_ARG;
    for (int i = 0; i < num_pairs; ++i)
        if (mapping[2 * i] < 0 || mapping[2 * i] >= src_blocks || mapping[2 * i + 1] < 0 ||
            mapping[2 * i + 1] >= dst_blocks)
            return PKVO_ERR_RANGE;
    for (int i = 0; i < num_pairs; ++i) {
        const uint16_t *src = src_cache + (int64_t)mapping[2 * i] * block_elems;
        uint16_t *dst = dst_cache + (int64_t)mapping[2 * i + 1] * block_elems;
        for (int64_t e = 0; e < block_elems; ++e)
            dst[e] = src[e];
    }
    return PKVO_OK;
}

/* ---- decode attention ([YK] 三, [FC] 二.2) ------------------------------ */

static int check_tables(const int32_t *block_tables, int max_blocks,
                        const int32_t *context_lens, int batch, int block_size,
                        int64_t num_blocks)
{
    for (int b = 0; b < batch; ++b) {
        int L = context_lens[b];
        if (L < 0 || (int64_t)L > (int64_t)max_blocks * block_size)
            return PKVO_ERR_RANGE;
        int used = (L + block_size - 1) / block_size;
        for (int i = 0; i < used; ++i) {
            int32_t id = block_tables[(int64_t)b * max_blocks + i];
            if (id < 0 || id >= num_blocks)
                return PKVO_ERR_RANGE;
        }
    }
    return PKVO_OK;
}

/*
 * Attention of query row q (query head h) over a sequence's logical tokens
 * [j0, j1), located through that sequence's block table: writes the max score m, the softmax normaliser
 * l = sum_j exp(s_j - m) and the normalised output o[d] = sum_j
 * exp(s_j - m) v_j[d] / l.  scores[] is caller scratch of j1-j0 entries;
 * it first holds the scores, then the weights.  An empty range gives m = -inf, l = 0, o = 0.
 */
static void attend_range(const uint16_t *q, const uint16_t *key_cache,
                         const uint16_t *value_cache, const int32_t *table,
                         int h, int j0, int j1, int Hq, int Hkv, int D,
                         int block_size, double scale, int dtype,
                         double *scores, double *m_out, double *l_out, double *o)
{
    int group = Hq / Hkv;
    int kvh = h / group;

    for (int d = 0; d < D; ++d)
        o[d] = 0.0;
    if (j1 <= j0) {
        *m_out = -INFINITY;
        *l_out = 0.0;
        return;
    }
    /* scores: s_j = scale * sum_d q[d] * K[block, offset, kvh, d] */
    for (int j = j0; j < j1; ++j) {
        int32_t block_id = table[j / block_size];
        int offset = j % block_size;
        const uint16_t *k = key_cache +
            (((int64_t)block_id * block_size + offset) * Hkv + kvh) * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += decode(q[d], dtype) * decode(k[d], dtype);
        scores[j - j0] = scale * dot;
    }
    /* softmax with the maximum subtracted */
    double m = -INFINITY;
    for (int j = j0; j < j1; ++j)
        if (scores[j - j0] > m)
            m = scores[j - j0];
    double l = 0.0;
    for (int j = j0; j < j1; ++j) {
        scores[j - j0] = exp(scores[j - j0] - m);   /* now the weight w_j */
        l += scores[j - j0];
    }
    /* weighted sum of V, normalised */
    for (int j = j0; j < j1; ++j) {
        int32_t block_id = table[j / block_size];
        int offset = j % block_size;
        const uint16_t *v = value_cache +
            (((int64_t)block_id * block_size + offset) * Hkv + kvh) * D;
        for (int d = 0; d < D; ++d)
            o[d] += scores[j - j0] * decode(v[d], dtype);
    }
    for (int d = 0; d < D; ++d)
        o[d] /= l;
    *m_out = m;
    *l_out = l;
}

/*
 * out[b, h, :] for every sequence b and query head h, in double, unrounded.
 * scratch must hold max_blocks * block_size doubles per thread (nthreads
 * slices).  Returns PKVO_ERR_RANGE (and writes nothing) if a context length
 * exceeds max_blocks * block_size or a used table entry is outside
 * [0, num_blocks).
 */
int pkvo_paged_attention_decode(const uint16_t *query, const uint16_t *key_cache,
                                const uint16_t *value_cache,
                                const int32_t *block_tables, int max_blocks,
                                const int32_t *context_lens, int batch, int Hq,
                                int Hkv, int D, int block_size, int64_t num_blocks,
                                double scale, int dtype, double *out,
                                double *scratch, int nthreads)
{
    if (batch < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 ||
        block_size <= 0 || max_blocks <= 0 || nthreads <= 0)
        return PKVO_ERR_ARG;
    int rc = check_tables(block_tables, max_blocks, context_lens, batch,
                          block_size, num_blocks);
    if (rc != PKVO_OK)
        return rc;
    int64_t span = (int64_t)max_blocks * block_size;
    int64_t pairs = (int64_t)batch * Hq;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int64_t bh = 0; bh < pairs; ++bh) {
        int b = (int)(bh / Hq), h = (int)(bh % Hq);
#ifdef _OPENMP
        double *sc = scratch + span * omp_get_thread_num();
#else
        double *sc = scratch;
#endif
        double m, l;
        attend_range(query + ((int64_t)b * Hq + h) * D, key_cache, value_cache,
                     block_tables + (int64_t)b * max_blocks, h, 0,
                     context_lens[b], Hq, Hkv, D, block_size, scale, dtype, sc,
                     &m, &l, out + bh * D);
    }
    return PKVO_OK;
}

/*
 * Chunked prefill: sequence b has query_start[b+1] - query_start[b] = C_b new
 * query tokens, the last C_b of its context_lens[b] = L_b cached tokens (their
 * K/V already written).  Query token i of b sits at logical position
 * p = L_b - C_b + i and attends over the cached tokens 0 .. p (causal):
 *   out[query_start[b] + i, h, :] = softmax_j<=p(scale * <q, K_j>) . V_j
 * query and out are [total_tokens, Hq, D].  Returns PKVO_ERR_RANGE if a
 * chunk is longer than its context or a context does not fit the table.
 */
int pkvo_paged_attention_prefill(const uint16_t *query, const int32_t *query_start,
                                 const uint16_t *key_cache, const uint16_t *value_cache,
                                 const int32_t *block_tables, int max_blocks,
                                 const int32_t *context_lens, int batch, int Hq, int Hkv, int D,
                                 int block_size, int64_t num_blocks, double scale, int dtype,
                                 double *out, double *scratch, int nthreads)
{
    if (batch < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 ||
        block_size <= 0 || max_blocks <= 0 || nthreads <= 0)
        return PKVO_ERR_ARG;
    int rc = check_tables(block_tables, max_blocks, context_lens, batch, block_size, num_blocks);
    if (rc != PKVO_OK)
        return rc;
    for (int b = 0; b < batch; ++b) {
        int C = query_start[b + 1] - query_start[b];
        if (C < 0 || C > context_lens[b])
            return PKVO_ERR_RANGE;
    }
    int64_t span = (int64_t)max_blocks * block_size;
    int64_t rows = (int64_t)query_start[batch] * Hq;
#pragma omp parallel for schedule(dynamic, 16) num_threads(nthreads)
    for (int64_t th = 0; th < rows; ++th) {
        int64_t t = th / Hq;
        int h = (int)(th % Hq);
        int b = 0;
        while (query_start[b + 1] <= t)     /* the sequence that owns token t */
            ++b;
        int i = (int)(t - query_start[b]);
        int C = query_start[b + 1] - query_start[b];
        int p = context_lens[b] - C + i;
#ifdef _OPENMP
        double *sc = scratch + span * omp_get_thread_num();
#else
        double *sc = scratch;
#endif
        double m, l;
        attend_range(query + th * D, key_cache, value_cache,
                     block_tables + (int64_t)b * max_blocks, h, 0, p + 1, Hq, Hkv, D,
                     block_size, scale, dtype, sc, &m, &l, out + th * D);
    }
    return PKVO_OK;
}

/*
 * Split-context form: for partition p of partition_tokens logical tokens,
 * m[b, h, p], l[b, h, p] and the normalised o[b, h, p, :] over the tokens
 * [p*P, min(L, (p+1)*P)).  Partitions past the end are empty (m = -inf,
 * l = 0, o = 0).  num_partitions partitions are produced per (b, h).
 */
int pkvo_paged_attention_partitions(const uint16_t *query, const uint16_t *key_cache,
                                    const uint16_t *value_cache,
                                    const int32_t *block_tables, int max_blocks,
                                    const int32_t *context_lens, int batch, int Hq,
                                    int Hkv, int D, int block_size, int64_t num_blocks,
                                    double scale, int dtype, int partition_tokens,
                                    int num_partitions, double *m_out, double *l_out,
                                    double *o_out, double *scratch)
{
    if (batch < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 ||
        block_size <= 0 || max_blocks <= 0 || partition_tokens <= 0 ||
        num_partitions <= 0)
        return PKVO_ERR_ARG;
    int rc = check_tables(block_tables, max_blocks, context_lens, batch,
                          block_size, num_blocks);
    if (rc != PKVO_OK)
        return rc;
    for (int b = 0; b < batch; ++b) {
        int L = context_lens[b];
        for (int h = 0; h < Hq; ++h) {
            for (int p = 0; p < num_partitions; ++p) {
                int64_t idx = ((int64_t)b * Hq + h) * num_partitions + p;
                int j0 = p * partition_tokens;
                int j1 = j0 + partition_tokens;
                if (j1 > L)
                    j1 = L;
                attend_range(query + ((int64_t)b * Hq + h) * D, key_cache, value_cache,
                             block_tables + (int64_t)b * max_blocks, h, j0, j1,
                             Hq, Hkv, D, block_size, scale, dtype, scratch,
                             &m_out[idx], &l_out[idx], o_out + idx * D);
            }
        }
    }
    return PKVO_OK;
}

/*
 * Log-sum-exp merge of the partitions of one (b, h) row set:
 *   M = max_p m_p,  w_p = exp(m_p - M) * l_p,
 *   out[:] = sum_p w_p * o_p[:] / sum_p w_p.
 * Empty partitions (l_p == 0) carry no weight.  rows = batch * Hq.
 */
void pkvo_lse_merge(const double *m, const double *l, const double *o,
                    int64_t rows, int num_partitions, int D, double *out)
{
    for (int64_t r = 0; r < rows; ++r) {
        const double *mr = m + r * num_partitions;
        const double *lr = l + r * num_partitions;
        double M = -INFINITY;
        for (int p = 0; p < num_partitions; ++p)
            if (lr[p] > 0.0 && mr[p] > M)
                M = mr[p];
        double den = 0.0;
        for (int d = 0; d < D; ++d)
            out[r * D + d] = 0.0;
        for (int p = 0; p < num_partitions; ++p) {
            if (!(lr[p] > 0.0))
                continue;
            double w = exp(mr[p] - M) * lr[p];
            den += w;
            for (int d = 0; d < D; ++d)
                out[r * D + d] += w * o[(r * num_partitions + p) * D + d];
        }
        if (den > 0.0)
            for (int d = 0; d < D; ++d)
                out[r * D + d] /= den;
    }
}
