/*
 * oracle.c -- plain, slow, fp64 CPU reference for paged attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this file:
 * only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg load it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it follows (vLLM V1 as described in "Inside vLLM: Anatomy of a
 * High-Throughput LLM Inference System"):
 *   - the KV cache is a pool of fixed 16-token blocks; a request's tokens live
 *     in the blocks its block table lists, in order (hn.213312.xyz restatement,
 *     section 一 "调度器"/"前向传播"; shengyayun.com blog, 关键实现细节 1-2);
 *   - every step builds a slot mapping and writes the step's new K/V into those
 *     slots before attention runs (hn.213312.xyz, section 一, "前向传播");
 *   - attention runs over all requests flattened into one "super-sequence";
 *     a prefill chunk attends causally to its request's cached context plus the
 *     chunk itself, and splitting a prompt into chunks must not change the
 *     result (hn.213312.xyz, section 二.1); prefix-cache hits reuse cached
 *     blocks as they are (section 二.2).
 *
 * Everything is the plain definition: gather the request's K/V through the
 * block table into contiguous arrays, then for each query row compute all
 * scores, subtract the maximum, exponentiate, normalise and take the weighted
 * sum of V -- one pass, no online softmax, no tiling, no splitting.
 * bf16 inputs are widened exactly to double; accumulation is in double.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* exact bf16 -> double (bf16 is the top half of an IEEE binary32) */
static double widen_bf16(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

double oracle_bf16_to_double(uint16_t bits) { return widen_bf16(bits); }

/* ------------------------------------------------------------------------
 * Slot mapping.  Token i of request r (0-based within this step) sits at
 * absolute position p = (seq_len - q_len) + i; its slot is
 * block_table[r][p / block_size] * block_size + p % block_size.
 * Returns 0, or -1 if a request has seq_len < q_len.
 * ---------------------------------------------------------------------- */
int oracle_slot_mapping(const int32_t *query_start_loc, const int32_t *seq_lens,
                        const int32_t *block_table, int64_t bt_stride, int32_t num_seqs,
                        int32_t block_size, int64_t *slot_mapping)
{
    for (int32_t r = 0; r < num_seqs; ++r) {
        int64_t q = (int64_t)query_start_loc[r + 1] - query_start_loc[r];
        int64_t c = (int64_t)seq_lens[r] - q;
        if (q < 0 || c < 0)
            return -1;
        for (int64_t i = 0; i < q; ++i) {
            int64_t p = c + i;
            int64_t blk = block_table[(int64_t)r * bt_stride + p / block_size];
            slot_mapping[query_start_loc[r] + i] = blk * block_size + p % block_size;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * KV write: for every token t with slot >= 0, copy the bit patterns of its
 * num_kv_heads x head_dim K and V rows into cache[slot / bs][h][slot % bs][:].
 * Cache layout: [num_blocks][num_kv_heads][block_size][head_dim].
 * New rows: token t, head h starts at k_new + t * row_stride + h * head_dim.
 * Returns 0, or -1 if a slot lies beyond the pool (nothing is written for it).
 * ---------------------------------------------------------------------- */
int oracle_kv_write(const uint16_t *k_new, const uint16_t *v_new, int64_t row_stride,
                    const int64_t *slot_mapping, int64_t num_tokens, uint16_t *k_cache,
                    uint16_t *v_cache, int64_t num_blocks, int32_t num_kv_heads, int32_t head_dim,
                    int32_t block_size)
{
    int rc = 0;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue; /* padding token */
        if (slot >= num_blocks * block_size) {
            rc = -1;
            continue;
        }
        int64_t blk = slot / block_size, off = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;
            int64_t src = t * row_stride + (int64_t)h * head_dim;
            memcpy(k_cache + dst, k_new + src, sizeof(uint16_t) * (size_t)head_dim);
            memcpy(v_cache + dst, v_new + src, sizeof(uint16_t) * (size_t)head_dim);
        }
    }
    return rc;
}

/* ------------------------------------------------------------------------
 * Gather: contiguous copy of one request's first seq_len tokens of one cache,
 * walking its block table (blocks 0 .. ceil(seq_len / bs) - 1 in order and
 * taking min(bs, seq_len - bs*b) rows from block b).
 * kv_head < 0: all heads, out is [seq_len][num_kv_heads][head_dim];
 * kv_head >= 0: that head only, out is [seq_len][head_dim].
 * Returns 0, or -1 on a block id outside the pool.
 * ---------------------------------------------------------------------- */
int oracle_gather_kv(const uint16_t *cache, int64_t num_blocks, int32_t num_kv_heads,
                     int32_t head_dim, int32_t block_size, const int32_t *bt_row, int64_t seq_len,
                     int32_t kv_head, uint16_t *out)
{
    int64_t nblk = (seq_len + block_size - 1) / block_size;
    int64_t j = 0;
    for (int64_t b = 0; b < nblk; ++b) {
        int64_t blk = bt_row[b];
        if (blk < 0 || blk >= num_blocks)
            return -1;
        int64_t rows = seq_len - b * block_size;
        if (rows > block_size)
            rows = block_size;
        for (int64_t o = 0; o < rows; ++o, ++j) {
            if (kv_head >= 0) {
                const uint16_t *src = cache + ((blk * num_kv_heads + kv_head) * block_size + o) * head_dim;
                memcpy(out + j * head_dim, src, sizeof(uint16_t) * (size_t)head_dim);
            } else {
                for (int32_t h = 0; h < num_kv_heads; ++h) {
                    const uint16_t *src = cache + ((blk * num_kv_heads + h) * block_size + o) * head_dim;
                    memcpy(out + (j * num_kv_heads + h) * head_dim, src,
                           sizeof(uint16_t) * (size_t)head_dim);
                }
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Block pack / unpack for moving KV between a prefill instance and a decode
 * instance (hn.213312.xyz section 二, item 5; shengyayun.com 关键实现细节
 * item 4): whole blocks are copied to and from a staging buffer.
 * A block is block_elems = num_kv_heads * block_size * head_dim contiguous
 * bf16 values of a cache, whatever the order inside it.
 * pack:   staging[i][0][:] = k_cache block ids[i], staging[i][1][:] = v block;
 *         an id outside [0, num_blocks) gives a zero entry.
 * unpack: k_cache block ids[i] = staging[i][0][:], v block = staging[i][1][:];
 *         an id outside the pool is skipped.
 * Both return the number of ids outside the pool.
 * ---------------------------------------------------------------------- */
int64_t oracle_kv_pack(const uint16_t *k_cache, const uint16_t *v_cache, int64_t num_blocks,
                       int64_t block_elems, const int32_t *ids, int64_t n, uint16_t *staging)
{
    int64_t bad = 0;
    for (int64_t i = 0; i < n; ++i) {
        uint16_t *dk = staging + (2 * i) * block_elems;
        uint16_t *dv = staging + (2 * i + 1) * block_elems;
        int64_t b = ids[i];
        if (b < 0 || b >= num_blocks) {
            memset(dk, 0, sizeof(uint16_t) * (size_t)block_elems);
            memset(dv, 0, sizeof(uint16_t) * (size_t)block_elems);
            ++bad;
            continue;
        }
        memcpy(dk, k_cache + b * block_elems, sizeof(uint16_t) * (size_t)block_elems);
        memcpy(dv, v_cache + b * block_elems, sizeof(uint16_t) * (size_t)block_elems);
    }
    return bad;
}

int64_t oracle_kv_unpack(const uint16_t *staging, const int32_t *ids, int64_t n, uint16_t *k_cache,
                         uint16_t *v_cache, int64_t num_blocks, int64_t block_elems)
{
    int64_t bad = 0;
    for (int64_t i = 0; i < n; ++i) {
        int64_t b = ids[i];
        if (b < 0 || b >= num_blocks) {
            ++bad;
            continue;
        }
        memcpy(k_cache + b * block_elems, staging + (2 * i) * block_elems,
               sizeof(uint16_t) * (size_t)block_elems);
        memcpy(v_cache + b * block_elems, staging + (2 * i + 1) * block_elems,
               sizeof(uint16_t) * (size_t)block_elems);
    }
    return bad;
}

/* ------------------------------------------------------------------------
 * Dense attention of one query row over n contiguous keys (the definition):
 *   s_j = scale * sum_d q[d] * K[j][d]
 *   w_j = exp(s_j - max_s) / sum_i exp(s_i - max_s)
 *   out = sum_j w_j * V[j]             lse = max_s + ln(sum_i exp(s_i - max_s))
 * K and V rows are ld elements apart.  n == 0 gives out = 0 and lse = -inf.
 * scratch must hold n doubles.  *wsum_err (if given) receives |sum_j w_j - 1|.
 * ---------------------------------------------------------------------- */
void oracle_attend_dense(const uint16_t *q, const uint16_t *K, const uint16_t *V, int64_t n,
                         int32_t head_dim, int64_t ld, double scale, double *out, double *lse,
                         double *scratch, double *wsum_err)
{
    for (int32_t d = 0; d < head_dim; ++d)
        out[d] = 0.0;
    if (n <= 0) {
        if (lse)
            *lse = -INFINITY;
        if (wsum_err)
            *wsum_err = 0.0;
        return;
    }
    double mx = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        double s = 0.0;
        for (int32_t d = 0; d < head_dim; ++d)
            s += widen_bf16(q[d]) * widen_bf16(K[j * ld + d]);
        s *= scale;
        scratch[j] = s;
        if (s > mx)
            mx = s;
    }
    double z = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        scratch[j] = exp(scratch[j] - mx);
        z += scratch[j];
    }
    double wsum = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        double w = scratch[j] / z;
        wsum += w;
        for (int32_t d = 0; d < head_dim; ++d)
            out[d] += w * widen_bf16(V[j * ld + d]);
    }
    if (lse)
        *lse = mx + log(z);
    if (wsum_err)
        *wsum_err = fabs(wsum - 1.0);
}

/* ------------------------------------------------------------------------
 * Merge of attention states over disjoint key sets (the split-KV reduce):
 * given per-part normalised outputs o_s and log-sum-exps lse_s,
 *   LSE = ln sum_s exp(lse_s),   out = sum_s exp(lse_s - LSE) * o_s.
 * This equals the (m, l, acc) form M = max m_s, l = sum_s l_s e^{m_s - M},
 * out = sum_s acc_s e^{m_s - M} / l with acc_s = o_s l_s, lse_s = m_s + ln l_s.
 * Parts with lse = -inf (no keys) carry no weight.
 * ---------------------------------------------------------------------- */
void oracle_merge_states(const double *o, const double *lse, int32_t num_parts, int32_t head_dim,
                         double *out, double *lse_out)
{
    double mx = -INFINITY;
    for (int32_t s = 0; s < num_parts; ++s)
        if (lse[s] > mx)
            mx = lse[s];
    for (int32_t d = 0; d < head_dim; ++d)
        out[d] = 0.0;
    if (mx == -INFINITY) {
        if (lse_out)
            *lse_out = -INFINITY;
        return;
    }
    double z = 0.0;
    for (int32_t s = 0; s < num_parts; ++s)
        z += exp(lse[s] - mx);
    for (int32_t s = 0; s < num_parts; ++s) {
        double w = exp(lse[s] - mx) / z;
        for (int32_t d = 0; d < head_dim; ++d)
            out[d] += w * o[(int64_t)s * head_dim + d];
    }
    if (lse_out)
        *lse_out = mx + log(z);
}

/* ------------------------------------------------------------------------
 * Attention for one step over the flattened super-sequence.
 *
 * Request r owns query rows [qsl[r], qsl[r+1]) and has seq_len L_r tokens in
 * the cache (this step's tokens already written).  Its cached context is
 * c_r = L_r - q_r.  Row i of the request sits at position p = c_r + i and its
 * query head h (kv head g = h / (Hq / Hkv)) attends keys 0 .. p of the
 * gathered K_r, V_r for head g.
 *
 * out: [T][Hq][D] doubles (or [n_list][Hq][D] when token_list is given),
 * lse: [T][Hq] (nullable).  max_wsum_err (nullable) gets the worst
 * |sum of softmax weights - 1| seen.  nthreads <= 0 uses every online core.
 * Returns 0, -1 on a bad block id or length, -2 on allocation failure.
 * ---------------------------------------------------------------------- */
typedef struct {
    const uint16_t *q, *k_cache, *v_cache;
    int32_t Hq, Hkv, D, bs;
    int64_t num_blocks;
    const int32_t *qsl, *seq_lens, *bt;
    int64_t bt_stride;
    int32_t num_seqs;
    double scale;
    double *out, *lse;
    const int32_t *token_list; /* NULL: every token */
    int32_t n_list;
    int64_t n_units;
    int64_t next_unit; /* atomically incremented */
    int error;
    double wsum_err;
    pthread_mutex_t mu;
} attn_ctx;

static int32_t request_of_token(const attn_ctx *c, int32_t t)
{
    int32_t lo = 0, hi = c->num_seqs - 1;
    while (lo < hi) { /* last r with qsl[r] <= t */
        int32_t mid = (lo + hi + 1) / 2;
        if (c->qsl[mid] <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo; /* the last such r owns t: empty requests before it are skipped */
}

/* unit = (request or listed token, kv head) */
static void run_unit(attn_ctx *c, int64_t unit, uint16_t **kbuf, uint16_t **vbuf, int64_t *cap,
                     double **scratch, double *worst)
{
    int32_t g = (int32_t)(unit % c->Hkv);
    int64_t item = unit / c->Hkv;
    int32_t r, t_begin, t_end;
    int64_t out_row0;
    if (c->token_list) {
        int32_t t = c->token_list[item];
        r = request_of_token(c, t);
        t_begin = t;
        t_end = t + 1;
        out_row0 = item;
    } else {
        r = (int32_t)item;
        t_begin = c->qsl[r];
        t_end = c->qsl[r + 1];
        out_row0 = t_begin;
    }
    int64_t q_len = (int64_t)c->qsl[r + 1] - c->qsl[r];
    int64_t L = c->seq_lens[r];
    int64_t ctx = L - q_len;
    if (q_len < 0 || ctx < 0) {
        c->error = -1;
        return;
    }
    if (t_end <= t_begin)
        return;
    /* keys needed: up to the last listed row's position */
    int64_t need = ctx + (t_end - c->qsl[r]);
    if (need > *cap) {
        free(*kbuf);
        free(*vbuf);
        free(*scratch);
        *kbuf = malloc(sizeof(uint16_t) * (size_t)need * c->D);
        *vbuf = malloc(sizeof(uint16_t) * (size_t)need * c->D);
        *scratch = malloc(sizeof(double) * (size_t)need);
        if (!*kbuf || !*vbuf || !*scratch) {
            c->error = -2;
            *cap = 0;
            return;
        }
        *cap = need;
    }
    const int32_t *row = c->bt + (int64_t)r * c->bt_stride;
    if (oracle_gather_kv(c->k_cache, c->num_blocks, c->Hkv, c->D, c->bs, row, need, g, *kbuf) ||
        oracle_gather_kv(c->v_cache, c->num_blocks, c->Hkv, c->D, c->bs, row, need, g, *vbuf)) {
        c->error = -1;
        return;
    }
    int32_t G = c->Hq / c->Hkv;
    for (int32_t t = t_begin; t < t_end; ++t) {
        int64_t p = ctx + (t - c->qsl[r]);
        int64_t orow = out_row0 + (t - t_begin);
        for (int32_t gi = 0; gi < G; ++gi) {
            int32_t h = g * G + gi;
            const uint16_t *qv = c->q + ((int64_t)t * c->Hq + h) * c->D;
            double err = 0.0;
            double lse;
            oracle_attend_dense(qv, *kbuf, *vbuf, p + 1, c->D, c->D, c->scale,
                                c->out + (orow * c->Hq + h) * c->D, &lse, *scratch, &err);
            if (c->lse)
                c->lse[orow * c->Hq + h] = lse;
            if (err > *worst)
                *worst = err;
        }
    }
}

static void *attn_worker(void *arg)
{
    attn_ctx *c = (attn_ctx *)arg;
    uint16_t *kbuf = NULL, *vbuf = NULL;
    double *scratch = NULL;
    int64_t cap = 0;
    double worst = 0.0;
    for (;;) {
        int64_t u = __atomic_fetch_add(&c->next_unit, 1, __ATOMIC_RELAXED);
        if (u >= c->n_units || c->error)
            break;
        run_unit(c, u, &kbuf, &vbuf, &cap, &scratch, &worst);
    }
    free(kbuf);
    free(vbuf);
    free(scratch);
    pthread_mutex_lock(&c->mu);
    if (worst > c->wsum_err)
        c->wsum_err = worst;
    pthread_mutex_unlock(&c->mu);
    return NULL;
}

int oracle_attention(const uint16_t *q, int32_t num_q_heads, const uint16_t *k_cache,
                     const uint16_t *v_cache, int64_t num_blocks, int32_t num_kv_heads,
                     int32_t head_dim, int32_t block_size, const int32_t *query_start_loc,
                     const int32_t *seq_lens, const int32_t *block_table, int64_t bt_stride,
                     int32_t num_seqs, double scale, const int32_t *token_list, int32_t n_list,
                     double *out, double *lse, double *max_wsum_err, int32_t nthreads)
{
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads)
        return -1;
    attn_ctx c;
    memset(&c, 0, sizeof c);
    c.q = q;
    c.k_cache = k_cache;
    c.v_cache = v_cache;
    c.Hq = num_q_heads;
    c.Hkv = num_kv_heads;
    c.D = head_dim;
    c.bs = block_size;
    c.num_blocks = num_blocks;
    c.qsl = query_start_loc;
    c.seq_lens = seq_lens;
    c.bt = block_table;
    c.bt_stride = bt_stride;
    c.num_seqs = num_seqs;
    c.scale = scale;
    c.out = out;
    c.lse = lse;
    c.token_list = token_list;
    c.n_list = n_list;
    c.n_units = (int64_t)(token_list ? n_list : num_seqs) * num_kv_heads;
    pthread_mutex_init(&c.mu, NULL);
    int64_t nt = nthreads > 0 ? nthreads : sysconf(_SC_NPROCESSORS_ONLN);
    if (nt < 1)
        nt = 1;
    if (nt > c.n_units)
        nt = c.n_units > 0 ? c.n_units : 1;
    pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nt);
    if (!th)
        return -2;
    for (int64_t i = 0; i < nt; ++i)
        pthread_create(&th[i], NULL, attn_worker, &c);
    for (int64_t i = 0; i < nt; ++i)
        pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&c.mu);
    if (max_wsum_err)
        *max_wsum_err = c.wsum_err;
    return c.error;
}

int oracle_num_cores(void) { return (int)sysconf(_SC_NPROCESSORS_ONLN); }
