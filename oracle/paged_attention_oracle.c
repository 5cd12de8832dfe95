/*
 * CPU oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, the smoke check and the bench's cpu_baseline / reference arm
 * may load this file's library.  It shares no code, header, table or helper
 * with the CUDA library in paged_kv_cache_393_b200/csrc, and it must never be
 * used as a fallback for it.
 *
 * What it computes (plain definition, double precision, no blocking or
 * reordering beyond the definition):
 *
 *   For each sequence b and query head h, with G = H / Hk and kv head
 *   kvh = h / G (contiguous query-head groups):
 *     1. Gather: for every logical token i < L_b, look up the physical block
 *        phys = block_tables[b][i / bs] and read row i % bs of that block:
 *            K_b[i][:] = key_cache  [phys][kvh][i % bs][:]
 *            V_b[i][:] = value_cache[phys][kvh][i % bs][:]
 *        (logical block to physical block through the per-sequence table: 5688vip ch. 4
 *        "PagedAttention：显存管理、分页机制、块大小选择", section
 *        "分页机制：块表与物理块的组织方式" and its block-table figure;
 *        lpnh.cn/news/2758356 §2.2 "Block Table"; lpnh.cn/news/1824136 §2.2
 *        item 3, addresses resolved while attention runs).
 *     2. Scores: s_i = scale * sum_d q[b][h][d] * K_b[i][d].
 *     3. Softmax with max subtraction: p_i = exp(s_i - max_j s_j) / Z,
 *        Z = sum_i exp(s_i - max_j s_j).
 *     4. Output: o[b][h][d] = sum_i p_i * V_b[i][d]   (returned in double).
 *
 *   Cache layout (the pages only say a block holds "block_size x num_kv_heads
 *   x head_dim", lpnh.cn/news/2758356 §2.1): [num_blocks][Hk][bs][D], fp16.
 *   The layout is isolated in kv_offset() below.
 *
 * fp16 inputs are decoded exactly to double by half_to_double(), written from
 * the IEEE 754 binary16 definition (1 sign bit, 5 exponent bits with bias 15,
 * 10 fraction bits).
 *
 * Status codes: 0 ok, -1 invalid argument (null pointer, bad shape, context
 * length <= 0 or beyond the table, physical block id out of range).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double mag;
    if (expo == 0)            /* zero or subnormal: frac * 2^-24 */
        mag = ldexp((double)frac, -24);
    else if (expo == 31)      /* infinity or NaN */
        mag = frac ? NAN : INFINITY;
    else                      /* normal: (1024 + frac) * 2^(expo - 25) */
        mag = ldexp((double)(1024 + frac), expo - 25);
    return sign ? -mag : mag;
}

/* Element offset of K/V row `off` of kv head `kvh` in physical block `phys`. */
static size_t kv_offset(long phys, int kvh, int off, int Hk, int bs, int D)
{
    return (((size_t)phys * Hk + kvh) * bs + off) * (size_t)D;
}

/*
 * Step 1 alone: gather sequence b's K and V rows of kv head kvh into the
 * contiguous arrays k_out[L][D], v_out[L][D] (double).  Exposed so the tests
 * can check the block-table translation by itself.
 */
int oracle_gather_kv(double *k_out, double *v_out,
                     const uint16_t *key_cache, const uint16_t *value_cache,
                     const int32_t *table_row, int L, int kvh,
                     int num_kv_heads, int block_size, int head_dim,
                     int max_blocks, int num_blocks)
{
    if (!k_out || !v_out || !key_cache || !value_cache || !table_row)
        return -1;
    if (L <= 0 || block_size <= 0 || head_dim <= 0 || num_kv_heads <= 0)
        return -1;
    if (kvh < 0 || kvh >= num_kv_heads)
        return -1;
    if ((long)L > (long)max_blocks * block_size)
        return -1;
    for (int i = 0; i < L; i++) {
        int logical = i / block_size;
        int off = i % block_size;
        long phys = table_row[logical];
        if (phys < 0 || phys >= num_blocks)
            return -1;
        size_t base = kv_offset(phys, kvh, off, num_kv_heads, block_size, head_dim);
        for (int d = 0; d < head_dim; d++) {
            k_out[(size_t)i * head_dim + d] = oracle_half_to_double(key_cache[base + d]);
            v_out[(size_t)i * head_dim + d] = oracle_half_to_double(value_cache[base + d]);
        }
    }
    return 0;
}

typedef struct {
    double *out;
    const uint16_t *q, *key_cache, *value_cache;
    const int32_t *block_tables, *context_lens;
    double scale;
    int block_size, num_kv_heads, num_seqs, num_heads, head_dim, max_blocks, num_blocks;
    long first, last;           /* range of (b, h) pairs for this worker */
    int status;
} oracle_job;

static void *oracle_worker(void *arg)
{
    oracle_job *job = (oracle_job *)arg;
    const int D = job->head_dim;
    const int G = job->num_heads / job->num_kv_heads;
    long max_len = (long)job->max_blocks * job->block_size;
    double *K = (double *)malloc(sizeof(double) * (size_t)max_len * D);
    double *V = (double *)malloc(sizeof(double) * (size_t)max_len * D);
    double *s = (double *)malloc(sizeof(double) * (size_t)max_len);
    if (!K || !V || !s) {
        job->status = -1;
        free(K); free(V); free(s);
        return NULL;
    }
    for (long pair = job->first; pair < job->last; pair++) {
        int b = (int)(pair / job->num_heads);
        int h = (int)(pair % job->num_heads);
        int kvh = h / G;
        int L = job->context_lens[b];
        const int32_t *row = job->block_tables + (size_t)b * job->max_blocks;
        if (oracle_gather_kv(K, V, job->key_cache, job->value_cache, row, L, kvh,
                             job->num_kv_heads, job->block_size, D,
                             job->max_blocks, job->num_blocks) != 0) {
            job->status = -1;
            break;
        }
        const uint16_t *qh = job->q + ((size_t)b * job->num_heads + h) * D;
        /* scores */
        double smax = -INFINITY;
        for (int i = 0; i < L; i++) {
            double dot = 0.0;
            for (int d = 0; d < D; d++)
                dot += oracle_half_to_double(qh[d]) * K[(size_t)i * D + d];
            s[i] = job->scale * dot;
            if (s[i] > smax)
                smax = s[i];
        }
        /* softmax with max subtraction */
        double Z = 0.0;
        for (int i = 0; i < L; i++) {
            s[i] = exp(s[i] - smax);
            Z += s[i];
        }
        /* weighted sum of V */
        double *o = job->out + ((size_t)b * job->num_heads + h) * D;
        for (int d = 0; d < D; d++) {
            double acc = 0.0;
            for (int i = 0; i < L; i++)
                acc += (s[i] / Z) * V[(size_t)i * D + d];
            o[d] = acc;
        }
    }
    free(K); free(V); free(s);
    return NULL;
}

/*
 * out[B][H][D] (double) = paged decode attention of q[B][H][D] (fp16 bits)
 * over the fp16 pools key_cache/value_cache[num_blocks][Hk][bs][D] through
 * block_tables[B][max_blocks] and context_lens[B].  nthreads <= 1 runs on the
 * calling thread; otherwise the (b, h) pairs are split into nthreads equal
 * contiguous ranges, one POSIX thread each.
 */
int oracle_paged_attention(double *out, const uint16_t *q,
                           const uint16_t *key_cache, const uint16_t *value_cache,
                           const int32_t *block_tables, const int32_t *context_lens,
                           double scale, int block_size, int num_kv_heads,
                           int num_seqs, int num_heads, int head_dim,
                           int max_blocks, int num_blocks, int nthreads)
{
    if (!out || !q || !key_cache || !value_cache || !block_tables || !context_lens)
        return -1;
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || max_blocks <= 0 || num_blocks <= 0)
        return -1;
    if (num_heads % num_kv_heads != 0)
        return -1;
    long pairs = (long)num_seqs * num_heads;
    if (pairs == 0)
        return 0;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > pairs)
        nthreads = (int)pairs;

    oracle_job *jobs = (oracle_job *)calloc((size_t)nthreads, sizeof(oracle_job));
    pthread_t *tids = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tids) {
        free(jobs); free(tids);
        return -1;
    }
    for (int t = 0; t < nthreads; t++) {
        oracle_job *j = &jobs[t];
        j->out = out; j->q = q; j->key_cache = key_cache; j->value_cache = value_cache;
        j->block_tables = block_tables; j->context_lens = context_lens;
        j->scale = scale; j->block_size = block_size; j->num_kv_heads = num_kv_heads;
        j->num_seqs = num_seqs; j->num_heads = num_heads; j->head_dim = head_dim;
        j->max_blocks = max_blocks; j->num_blocks = num_blocks;
        j->first = pairs * t / nthreads;
        j->last = pairs * (t + 1) / nthreads;
        j->status = 0;
    }
    int status = 0;
    if (nthreads == 1) {
        oracle_worker(&jobs[0]);
    } else {
        int started = 0;
        for (int t = 0; t < nthreads; t++) {
            if (pthread_create(&tids[t], NULL, oracle_worker, &jobs[t]) != 0) {
                /* run the rest inline if a thread cannot be created */
                for (int u = t; u < nthreads; u++)
                    oracle_worker(&jobs[u]);
                break;
            }
            started++;
        }
        for (int t = 0; t < started; t++)
            pthread_join(tids[t], NULL);
    }
    for (int t = 0; t < nthreads; t++)
        if (jobs[t].status != 0)
            status = -1;
    free(jobs);
    free(tids);
    return status;
}
