/*
 * oracle.c -- plain, slow fp64 reference for single-token (decode) attention
 * over a compressed or shared KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load or call this code.  It
 * shares nothing with the CUDA library (no headers, helpers or tables), and
 * the library never calls it.
 *
 * What it computes (one query token per sequence):
 *
 *   MLA explainer (mlqm.cn/news/371735), section 2.3, the attention formula
 *     o_{t,i} = sum_j softmax_j( q_{t,i}^T k_{j,i} / sqrt(d) ) v^C_{j,i}
 *   with section 2.2's concatenations q = [q^C ; q^R], k = [k^C ; k^R].
 *   MLRA page (aitntnews.com newId=23265), "Moving the sum outside": absorbed
 *   MLA is one wide MQA head whose key is [latent ; rope key] and whose value
 *   is the latent itself; MLRA attends each latent branch on its own and sums
 *   the branch outputs after attention.
 *   GLA page (jsbsmhs.com/zixun/902167), "Grouped Latent Attention": each
 *   latent head serves one group of query heads.
 *   MLRA page, the GQA and MQA bullets: a group of query heads (or all of
 *   them) shares one K/V head.
 *   GTA/GLA page (jsbsmhs.com/zixun/902167), "Grouped Tied Attention": the
 *   heads of a group share one key-value state, tied: the cached vector is
 *   both the key and the value (MFA page, jsqmd.com/news/79551: key reuse,
 *   MFA-KR, read as the same tie on MFA's single wide head).
 *
 * Readings where the pages are silent:
 *   - the 1/sqrt(d) factor is the caller's sm_scale and multiplies the whole
 *     score (nope + rope part);
 *   - lse is the natural log of sum_j exp(sm_scale * q.k_j);
 *   - an empty sequence gives o = 0 and lse = -inf;
 *   - MLRA keeps one lse per (head, branch) and sums the normalised branch
 *     outputs in latent space;
 *   - GLA: head h belongs to group h / (H / G); the RoPE key is shared by all
 *     groups; MLRA: every head attends every branch with its own query slice;
 *   - GTA: head h uses tied state h / (H / G), no separate rope part.
 *
 * Per (sequence b, head h[, branch r]) the softmax is taken the plain way, in
 * two passes over the scores: s_j for every cached token, m = max_j s_j,
 * Z = sum_j exp(s_j - m), o = sum_j exp(s_j - m) v_j / Z, lse = m + ln Z.
 * Every input element is widened to double before use; all arithmetic is in
 * double.  Work items (b, h) are independent and are spread over threads;
 * nothing inside an item is reordered.
 *
 * Cache layouts: latent pool [num_pages][page_size][num_kv*d_nope + d_rope],
 * row = [c_0 | ... | c_{num_kv-1} | k_rope]; GQA/MQA pool
 * [num_pages][2 (K,V)][page_size][num_kv][d_nope]; GTA pool (one tied plane)
 * [num_pages][page_size][num_kv][d_nope].  Token j of sequence b is
 * slot j % page_size of page block_table[b][j / page_size] (contiguous mode:
 * page b*max_pages_per_seq + j / page_size).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_GQA = 0, ORC_MQA = 1, ORC_MLA = 2, ORC_GLA = 3, ORC_MLRA = 4, ORC_GTA = 5 };
enum { ORC_BF16 = 0, ORC_F64 = 1 };

typedef struct {
    int32_t variant;
    int32_t batch, num_q_heads, num_kv, d_nope, d_rope;
    int32_t page_size, max_pages_per_seq, num_pages;
    int32_t paged;
} orc_shape;

typedef struct {
    const orc_shape *s;
    int elem_type;
    const void *q_nope, *q_rope, *kv;
    const int32_t *block_table, *seq_lens, *b_list, *h_list;
    int32_t n_b, n_h;
    double sm_scale;
    double *out, *lse;
    int32_t nthreads, tid;
    int status;
    int32_t branch_out;   /* MLRA: write the branch outputs side by side instead of their sum */
} orc_job;

/* Widen one input element to double (bf16 bits are the top half of a float). */
static double elem(const void *base, int type, size_t i)
{
    if (type == ORC_F64)
        return ((const double *)base)[i];
    uint32_t u = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int is_latent(int v) { return v == ORC_MLA || v == ORC_GLA || v == ORC_MLRA; }

/* Planes of a GQA/MQA page: K and V, or one tied plane (GTA). */
static size_t planes(const orc_shape *s) { return s->variant == ORC_GTA ? 1 : 2; }

/* Physical page of the i-th logical page of sequence b. */
static int64_t page_of(const orc_job *J, int b, int i)
{
    const orc_shape *s = J->s;
    if (!s->paged)
        return (int64_t)b * s->max_pages_per_seq + i;
    return J->block_table[(size_t)b * s->max_pages_per_seq + i];
}

/* Element offset of key element d (0 <= d < d_nope + d_rope) of token slot
 * (page, slot) for unit u (KV head, latent group or branch). */
static size_t key_index(const orc_shape *s, int64_t page, int slot, int u, int d)
{
    size_t dn = (size_t)s->d_nope;
    if (is_latent(s->variant)) {
        size_t row = (size_t)s->num_kv * dn + (size_t)s->d_rope;
        size_t base = ((size_t)page * s->page_size + slot) * row;
        if ((size_t)d < dn)
            return base + (size_t)u * dn + d;
        return base + (size_t)s->num_kv * dn + (d - dn);
    }
    return (((size_t)page * planes(s) + 0) * s->page_size + slot) * s->num_kv * dn + (size_t)u * dn + d;
}

/* Element offset of value element d of token slot (page, slot), unit u. */
static size_t value_index(const orc_shape *s, int64_t page, int slot, int u, int d)
{
    size_t dn = (size_t)s->d_nope;
    if (is_latent(s->variant)) {
        size_t row = (size_t)s->num_kv * dn + (size_t)s->d_rope;
        return ((size_t)page * s->page_size + slot) * row + (size_t)u * dn + d;
    }
    /* the V plane; a tied pool has one plane, its vector is the value too */
    return (((size_t)page * planes(s) + planes(s) - 1) * s->page_size + slot) * s->num_kv * dn + (size_t)u * dn + d;
}

/* Attention of one query row against all cached tokens of sequence b through
 * unit u.  q_row indexes q_nope/q_rope in units of one query row.  Writes
 * dv = d_nope doubles to o and returns lse through *lse. */
static int attend(const orc_job *J, int b, int u, size_t q_row, double *o, double *lse,
                  double *q, double *k, double *sc)
{
    const orc_shape *s = J->s;
    int dn = s->d_nope, dr = s->d_rope, dk = dn + dr;
    int L = J->seq_lens[b];
    for (int d = 0; d < dn; ++d)
        q[d] = elem(J->q_nope, J->elem_type, q_row * dn + d);
    for (int d = 0; d < dr; ++d)
        q[dn + d] = elem(J->q_rope, J->elem_type, q_row * dr + d);

    for (int d = 0; d < dn; ++d)
        o[d] = 0.0;
    if (L <= 0) {
        *lse = -INFINITY;
        return 0;
    }

    /* pass 1: scores */
    for (int j = 0; j < L; ++j) {
        int64_t page = page_of(J, b, j / s->page_size);
        int slot = j % s->page_size;
        if (page < 0 || page >= s->num_pages)
            return -1;
        for (int d = 0; d < dk; ++d)
            k[d] = elem(J->kv, J->elem_type, key_index(s, page, slot, u, d));
        double dot = 0.0;
        for (int d = 0; d < dk; ++d)
            dot += q[d] * k[d];
        sc[j] = J->sm_scale * dot;
    }
    double m = sc[0];
    for (int j = 1; j < L; ++j)
        if (sc[j] > m)
            m = sc[j];
    double Z = 0.0;
    for (int j = 0; j < L; ++j)
        Z += exp(sc[j] - m);

    /* pass 2: weighted sum of values */
    for (int j = 0; j < L; ++j) {
        int64_t page = page_of(J, b, j / s->page_size);
        int slot = j % s->page_size;
        double p = exp(sc[j] - m) / Z;
        for (int d = 0; d < dn; ++d)
            o[d] += p * elem(J->kv, J->elem_type, value_index(s, page, slot, u, d));
    }
    *lse = m + log(Z);
    return 0;
}

static void *worker(void *arg)
{
    orc_job *J = (orc_job *)arg;
    const orc_shape *s = J->s;
    int H = s->num_q_heads, dn = s->d_nope, dk = s->d_nope + s->d_rope;
    int maxL = 0;
    for (int i = 0; i < J->n_b; ++i)
        if (J->seq_lens[J->b_list[i]] > maxL)
            maxL = J->seq_lens[J->b_list[i]];
    double *q = malloc(sizeof(double) * (size_t)(dk > 0 ? dk : 1));
    double *k = malloc(sizeof(double) * (size_t)(dk > 0 ? dk : 1));
    double *o = malloc(sizeof(double) * (size_t)(dn > 0 ? dn : 1));
    double *sc = malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
    if (!q || !k || !o || !sc) {
        J->status = -2;
        goto done;
    }
    int nh = J->n_h;
    size_t items = (size_t)J->n_b * nh;
    for (size_t it = (size_t)J->tid; it < items; it += (size_t)J->nthreads) {
        int bi = (int)(it / nh), hi = (int)(it % nh);
        int b = J->b_list[bi];
        int h = J->h_list ? J->h_list[hi] : hi;
        double *dst = J->out + ((size_t)bi * nh + hi) * dn;
        if (s->variant == ORC_MLRA) {
            int R = s->num_kv;
            if (J->branch_out)
                dst = J->out + ((size_t)bi * nh + hi) * R * dn;
            else
                for (int d = 0; d < dn; ++d)
                    dst[d] = 0.0;
            for (int r = 0; r < R; ++r) {
                double l;
                size_t q_row = ((size_t)b * H + h) * R + r;
                if (attend(J, b, r, q_row, o, &l, q, k, sc)) {
                    J->status = -1;
                    goto done;
                }
                /* branch outputs side by side, or their sum */
                for (int d = 0; d < dn; ++d) {
                    if (J->branch_out)
                        dst[(size_t)r * dn + d] = o[d];
                    else
                        dst[d] += o[d];
                }
                J->lse[((size_t)bi * nh + hi) * R + r] = l;
            }
        } else {
            int u = 0;
            if (s->variant != ORC_MLA)
                u = h / (H / s->num_kv);
            double l;
            if (attend(J, b, u, (size_t)b * H + h, dst, &l, q, k, sc)) {
                J->status = -1;
                goto done;
            }
            J->lse[(size_t)bi * nh + hi] = l;
        }
    }
done:
    free(q);
    free(k);
    free(o);
    free(sc);
    return NULL;
}

/*
 * Decode attention for the sequences listed in b_list (n_b of them) and the
 * heads listed in h_list (n_h of them; h_list = NULL means all H heads).
 * elem_type: 0 = inputs are bf16 bit patterns (uint16), 1 = inputs are double.
 * out: [n_b][n_h][d_nope] (MLRA: sum over branches, or with branch_out the
 * R branch outputs [n_b][n_h][R][d_nope]); lse: [n_b][n_h] (MLRA
 * [n_b][n_h][R]).  Returns 0, -1 for a page id outside the pool, -2 when out
 * of memory, -3 for an invalid shape.
 */
int orc_decode(const orc_shape *s, int32_t elem_type, const void *q_nope, const void *q_rope,
               const void *kv, const int32_t *block_table, const int32_t *seq_lens,
               double sm_scale, const int32_t *b_list, int32_t n_b, const int32_t *h_list,
               int32_t n_h, double *out, double *lse, int32_t nthreads, int32_t branch_out)
{
    if (!s || s->variant < 0 || s->variant > ORC_GTA || s->num_kv <= 0 || s->num_q_heads <= 0 ||
        s->d_nope <= 0 || s->d_rope < 0 || s->page_size <= 0)
        return -3;
    if (s->variant != ORC_MLA && s->variant != ORC_MLRA && s->num_q_heads % s->num_kv)
        return -3;
    if (s->variant == ORC_MLA && s->num_kv != 1)
        return -3;
    if (!is_latent(s->variant) && s->d_rope != 0)
        return -3;
    for (int i = 0; i < n_b; ++i) {
        int b = b_list[i];
        if (b < 0 || b >= s->batch || seq_lens[b] > s->max_pages_per_seq * s->page_size)
            return -3;
    }
    if (!h_list)
        n_h = s->num_q_heads;
    for (int i = 0; h_list && i < n_h; ++i)
        if (h_list[i] < 0 || h_list[i] >= s->num_q_heads)
            return -3;
    if (nthreads < 1)
        nthreads = 1;
    orc_job *jobs = calloc((size_t)nthreads, sizeof(orc_job));
    pthread_t *th = calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return -2;
    }
    for (int t = 0; t < nthreads; ++t) {
        orc_job J = {s, elem_type, q_nope, q_rope, kv, block_table, seq_lens, b_list, h_list,
                     n_b, n_h, sm_scale, out, lse, nthreads, t, 0, branch_out};
        jobs[t] = J;
    }
    int started = 0;
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, worker, &jobs[t]) != 0)
            break;
        started = t;
    }
    /* threads that failed to start: their items run here, one after another */
    for (int t = started + 1; t < nthreads; ++t)
        worker(&jobs[t]);
    worker(&jobs[0]);
    for (int t = 1; t <= started; ++t)
        pthread_join(th[t], NULL);
    int status = 0;
    for (int t = 0; t < nthreads; ++t)
        if (jobs[t].status)
            status = jobs[t].status;
    free(jobs);
    free(th);
    return status;
}

/*
 * Merge of attention results over disjoint parts of one context (the split
 * combine).  With lse_p the log-sum-exp of part p and o_p its normalised
 * output, the whole context has lse = ln sum_p exp(lse_p) and
 * o = sum_p exp(lse_p - lse) o_p.  A part with lse = -inf (empty) has weight
 * 0; if every part is empty the result is o = 0, lse = -inf.
 * o_s: [n_part][rows][dv], lse_s: [n_part][rows]; o: [rows][dv], lse: [rows].
 */
void orc_merge(int32_t n_part, int32_t rows, int32_t dv, const double *o_s, const double *lse_s,
               double *o, double *lse)
{
    for (int r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int p = 0; p < n_part; ++p)
            if (lse_s[(size_t)p * rows + r] > m)
                m = lse_s[(size_t)p * rows + r];
        for (int d = 0; d < dv; ++d)
            o[(size_t)r * dv + d] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double Z = 0.0;
        for (int p = 0; p < n_part; ++p)
            Z += exp(lse_s[(size_t)p * rows + r] - m);
        double total = m + log(Z);
        for (int p = 0; p < n_part; ++p) {
            double w = exp(lse_s[(size_t)p * rows + r] - total);
            for (int d = 0; d < dv; ++d)
                o[(size_t)r * dv + d] += w * o_s[((size_t)p * rows + r) * dv + d];
        }
        lse[r] = total;
    }
}
