/*
 * Plain CPU oracle for paged-KV attention, in fp64.
 *
 * TEST INFRASTRUCTURE ONLY. It is called only by tests/, by the smoke check
 * in __graft_entry__.py and by the cpu_baseline and reference legs of
 * bench.py. It shares no code, header or constant with the CUDA library
 * under paged_kv_cache_366_b200/csrc, and neither one includes or links the
 * other. Product code never reaches it.
 *
 * What it computes, and where the pages state it:
 *
 *  - The cache is a pool of fixed-size blocks. Logical block i of a
 *    sequence lives in physical block table[i] ("vLLM and PagedAttention",
 *    ai.zenoagi.com, §2 "The PagedAttention Solution"; "vLLM — PagedAttention
 *    and Continuous Batching", s-samarth.github.io, §2.2). Logical position p
 *    is therefore slot table[p / bs] * bs + p % bs. The "100th token needs
 *    the 7th block" example in the first of these pins it
 *    (tests/golden/page_examples.txt).
 *  - Pool layout is [num_blocks, block_size, kv_heads, head_dim], from the
 *    kernel sketch's key_cache/value_cache comment ("vLLM and PagedAttention"
 *    §2 "Reworking the Attention Computation").
 *  - Paging changes where K and V live, not what attention computes. The
 *    kernel "indexes through a page table" (s-samarth §2.4). So the oracle
 *    gathers each sequence's blocks into contiguous K/V and runs textbook
 *    softmax attention on them, exp(s - max) / sum, in fp64.
 *  - Query head h reads KV head h / (H / Hk). The pages are silent here;
 *    contiguous groups is the reading taken.
 *  - Decode attends over all context_len tokens, including the one written
 *    this step. Prefill query j of a chunk of q_len tokens sits at absolute
 *    position (context_len - q_len) + j and attends to keys 0..position
 *    inclusive. Chunked prefill is described in s-samarth §5 and in
 *    "How vLLM Works?", peterindia.net, §04.
 *  - The cache write copies each new token's K/V row into its slot. A
 *    negative slot is padding and is skipped. This is the on-demand block
 *    use of "vLLM and PagedAttention" §2 and "How vLLM Works?" §03.
 *
 * bf16 inputs are widened exactly to fp64 (bf16 bits << 16 is an fp32 value).
 *
 * pa_oracle_set_mutation() plants known mistakes so the tests can show that
 * the pins catch them. Its default (0) is the oracle proper.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_FP8_E4M3 = 2 };

enum {
    MUT_NONE = 0,
    MUT_GQA_MODULO = 1,      /* kv head = h % Hk instead of h / G            */
    MUT_IGNORE_TABLE = 2,    /* physical block = logical block index          */
    MUT_NO_SCALE = 3,        /* softmax scale dropped                         */
    MUT_CAUSAL_EXCL = 4,     /* prefill query does not see its own key        */
    MUT_DROP_PARTIAL = 5,    /* last partly filled block skipped              */
    MUT_V_FROM_K = 6,        /* values read from the key cache                */
    MUT_WRITE_NEXT = 7,      /* cache write lands one slot later              */
    MUT_OFFSET_REV = 8,      /* row inside a block reversed                   */
    MUT_NO_DENOM = 9,        /* softmax denominator dropped                   */
    MUT_ZERO_OFFSET = 10,    /* prefill chunk placed at context offset 0      */
};

static int g_mutation = MUT_NONE;

void pa_oracle_set_mutation(int m) { g_mutation = m; }
int pa_oracle_get_mutation(void) { return g_mutation; }

/*
 * FP8 E4M3 (the "fn" variant: 1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits, no infinities, S.1111.111 is NaN, largest finite 448), written from
 * the format's definition. Codes 0x01..0x07 are subnormals k * 2^-9.
 */
double pa_oracle_e4m3_decode(uint8_t code)
{
    int sign = code >> 7, e = (code >> 3) & 0xF, m = code & 7;
    double v;
    if (e == 0xF && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Round a float to E4M3: nearest, ties to even; finite values past 448 saturate to 448. */
uint8_t pa_oracle_e4m3_encode(float f)
{
    if (isnan(f))
        return 0x7F;
    uint8_t sign = signbit(f) ? 0x80 : 0;
    double a = fabs((double)f);
    if (a >= 448.0)
        return sign | 0x7E;
    /* every representable magnitude is a multiple of its binade's quantum */
    int e;
    frexp(a, &e); /* a = f * 2^e with f in [0.5, 1): binade 2^(e-1) */
    int be = e - 1;
    if (be < -6)
        be = -6; /* subnormals share the quantum of the lowest normal binade */
    double q = ldexp(1.0, be - 3);
    double n = a / q; /* exact: q is a power of two */
    double r = floor(n);
    double frac = n - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) == 1.0))
        r += 1.0;
    double v = r * q; /* the rounded magnitude */
    if (v >= 448.0)
        return sign | 0x7E;
    if (v == 0.0)
        return sign;
    if (v < ldexp(1.0, -6))
        return sign | (uint8_t)(v / ldexp(1.0, -9));
    int ve;
    double vf = frexp(v, &ve); /* v = vf * 2^ve, vf in [0.5, 1) */
    int exp_field = ve - 1 + 7;
    int mant = (int)((vf * 2.0 - 1.0) * 8.0);
    return sign | (uint8_t)(exp_field << 3) | (uint8_t)mant;
}

static double load_elem(const void *base, long idx, int dtype)
{
    if (dtype == ORACLE_FP8_E4M3)
        return pa_oracle_e4m3_decode(((const uint8_t *)base)[idx]);
    if (dtype == ORACLE_BF16) {
        uint32_t u = (uint32_t)((const uint16_t *)base)[idx] << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return (double)((const float *)base)[idx];
}

/* Blocks needed to hold n tokens. */
long pa_oracle_blocks_for(long n_tokens, int block_size)
{
    return (n_tokens + block_size - 1) / block_size;
}

/* Flat slot of logical position p through one sequence's table row. */
long pa_oracle_slot_of(const int32_t *table_row, long p, int block_size)
{
    long logical_block = p / block_size;
    long offset = p % block_size;
    long physical_block = table_row[logical_block];
    if (g_mutation == MUT_IGNORE_TABLE)
        physical_block = logical_block;
    if (g_mutation == MUT_OFFSET_REV)
        offset = block_size - 1 - offset;
    return physical_block * block_size + offset;
}

/*
 * Gather sequence `seq`'s first n tokens for KV head hk into contiguous
 * Kc[n][D] and Vc[n][D] (fp64). Returns 0, or -1 if the table names a
 * block outside the pool.
 */
int pa_oracle_gather(double *Kc, double *Vc, const void *k_cache, const void *v_cache, int dtype,
                     const int32_t *block_tables, int max_blocks_per_seq, int seq, long n,
                     int num_kv_heads, int kv_head, int head_dim, int block_size, long num_blocks)
{
    const int32_t *row = block_tables + (long)seq * max_blocks_per_seq;
    if (pa_oracle_blocks_for(n, block_size) > max_blocks_per_seq)
        return -1;
    for (long p = 0; p < n; ++p) {
        long slot = pa_oracle_slot_of(row, p, block_size);
        if (slot < 0 || slot >= num_blocks * block_size)
            return -1;
        long base = (slot * num_kv_heads + kv_head) * head_dim;
        const void *vsrc = (g_mutation == MUT_V_FROM_K) ? k_cache : v_cache;
        for (int d = 0; d < head_dim; ++d) {
            Kc[p * head_dim + d] = load_elem(k_cache, base + d, dtype);
            Vc[p * head_dim + d] = load_elem(vsrc, base + d, dtype);
        }
    }
    return 0;
}

/* Softmax attention of one query over keys 0..n-1 of contiguous Kc/Vc. */
static void attend(double *o, const double *qv, const double *Kc, const double *Vc, long n, int D,
                   double scale, double *s)
{
    for (int d = 0; d < D; ++d)
        o[d] = 0.0;
    if (n <= 0)
        return;
    if (g_mutation == MUT_NO_SCALE)
        scale = 1.0;
    double m = -INFINITY;
    for (long p = 0; p < n; ++p) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += qv[d] * Kc[p * D + d];
        s[p] = scale * dot;
        if (s[p] > m)
            m = s[p];
    }
    double den = 0.0;
    for (long p = 0; p < n; ++p) {
        double w = exp(s[p] - m);
        den += w;
        for (int d = 0; d < D; ++d)
            o[d] += w * Vc[p * D + d];
    }
    if (g_mutation == MUT_NO_DENOM)
        den = 1.0;
    for (int d = 0; d < D; ++d)
        o[d] /= den;
}

static int kv_head_of(int h, int num_heads, int num_kv_heads)
{
    if (g_mutation == MUT_GQA_MODULO)
        return h % num_kv_heads;
    return h / (num_heads / num_kv_heads);
}

/* Tokens of a context the attention reads (the mutation drops the partial block). */
static long readable_tokens(long c, int block_size)
{
    if (g_mutation == MUT_DROP_PARTIAL)
        return (c / block_size) * block_size;
    return c;
}

static int set_threads(int num_threads)
{
#ifdef _OPENMP
    if (num_threads > 0)
        return num_threads;
    return omp_get_max_threads();
#else
    (void)num_threads;
    return 1;
#endif
}

/*
 * Decode: one query token per sequence, q [B][H][D] -> out [B][H][D] (fp64).
 * Returns 0, -1 for a table entry outside the pool, -2 for bad arguments.
 */
int pa_oracle_decode(double *out, const void *q, const void *k_cache, const void *v_cache, int dtype,
                     const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                     int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                     long num_blocks, double scale, int num_threads)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0)
        return -2;
    int nt = set_threads(num_threads);
    int status = 0;
    long units = (long)num_seqs * num_kv_heads;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (long u = 0; u < units; ++u) {
        int b = (int)(u / num_kv_heads), hk = (int)(u % num_kv_heads);
        long c = context_lens[b];
        double *Kc = malloc(sizeof(double) * (size_t)(c > 0 ? c : 1) * head_dim);
        double *Vc = malloc(sizeof(double) * (size_t)(c > 0 ? c : 1) * head_dim);
        double *s = malloc(sizeof(double) * (size_t)(c > 0 ? c : 1));
        double *qv = malloc(sizeof(double) * (size_t)head_dim);
        int rc = (c < 0) ? -2 : pa_oracle_gather(Kc, Vc, k_cache, v_cache, dtype, block_tables,
                                                  max_blocks_per_seq, b, c, num_kv_heads, hk,
                                                  head_dim, block_size, num_blocks);
        if (rc) {
#pragma omp critical
            status = rc;
        } else {
            for (int h = 0; h < num_heads; ++h) {
                if (kv_head_of(h, num_heads, num_kv_heads) != hk)
                    continue;
                long qbase = ((long)b * num_heads + h) * head_dim;
                for (int d = 0; d < head_dim; ++d)
                    qv[d] = load_elem(q, qbase + d, dtype);
                attend(out + qbase, qv, Kc, Vc, readable_tokens(c, block_size), head_dim, scale, s);
            }
        }
        free(Kc);
        free(Vc);
        free(s);
        free(qv);
    }
    return status;
}

/*
 * Prefill chunk: q [T][H][D] holds the chunk tokens of every sequence,
 * sequence b owning rows cu_q_lens[b] .. cu_q_lens[b+1]-1. context_lens
 * include the chunk. If `rows` is NULL every row is computed and
 * out is [T][H][D]. Otherwise out is [n_rows][H][D], holding the listed
 * global rows in order. Returns 0, -1 or -2 as decode does.
 */
static int prefill_impl(double *out, const void *q, int q_dtype, const void *k_cache, const void *v_cache,
                        int kv_dtype, double k_scale, double v_scale, const int32_t *block_tables,
                        int max_blocks_per_seq, const int32_t *cu_q_lens, const int32_t *context_lens,
                        int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                        long num_blocks, double scale, const int32_t *rows, long n_rows, int num_threads)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0)
        return -2;
    long total = cu_q_lens[num_seqs];
    if (rows == NULL)
        n_rows = total;
    for (long i = 0; i < n_rows; ++i) {
        long r = rows ? rows[i] : i;
        if (r < 0 || r >= total)
            return -2;
    }
    int nt = set_threads(num_threads);
    int status = 0;
    long units = (long)num_seqs * num_kv_heads;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (long u = 0; u < units; ++u) {
        int b = (int)(u / num_kv_heads), hk = (int)(u % num_kv_heads);
        long q0 = cu_q_lens[b], q1 = cu_q_lens[b + 1];
        long c = context_lens[b];
        long offset = c - (q1 - q0);
        if (g_mutation == MUT_ZERO_OFFSET)
            offset = 0;
        int wanted = 0;
        for (long i = 0; i < n_rows && !wanted; ++i) {
            long r = rows ? rows[i] : i;
            wanted = (r >= q0 && r < q1);
        }
        if (!wanted)
            continue;
        if (c < 0 || offset < 0) {
#pragma omp critical
            status = -2;
            continue;
        }
        double *Kc = malloc(sizeof(double) * (size_t)(c > 0 ? c : 1) * head_dim);
        double *Vc = malloc(sizeof(double) * (size_t)(c > 0 ? c : 1) * head_dim);
        double *s = malloc(sizeof(double) * (size_t)(c > 0 ? c : 1));
        double *qv = malloc(sizeof(double) * (size_t)head_dim);
        int rc = pa_oracle_gather(Kc, Vc, k_cache, v_cache, kv_dtype, block_tables, max_blocks_per_seq, b,
                                  c, num_kv_heads, hk, head_dim, block_size, num_blocks);
        if (rc) {
#pragma omp critical
            status = rc;
        } else {
            if (kv_dtype == ORACLE_FP8_E4M3) {
                for (long i = 0; i < c * head_dim; ++i) {
                    Kc[i] *= k_scale;
                    Vc[i] *= v_scale;
                }
            }
            for (long i = 0; i < n_rows; ++i) {
                long r = rows ? rows[i] : i;
                if (r < q0 || r >= q1)
                    continue;
                long pos = offset + (r - q0);
                long n_keys = pos + 1;
                if (g_mutation == MUT_CAUSAL_EXCL)
                    n_keys = pos;
                long readable = readable_tokens(c, block_size);
                if (n_keys > readable)
                    n_keys = readable;
                for (int h = 0; h < num_heads; ++h) {
                    if (kv_head_of(h, num_heads, num_kv_heads) != hk)
                        continue;
                    long qbase = (r * num_heads + h) * (long)head_dim;
                    for (int d = 0; d < head_dim; ++d)
                        qv[d] = load_elem(q, qbase + d, q_dtype);
                    attend(out + (i * num_heads + h) * (long)head_dim, qv, Kc, Vc, n_keys, head_dim,
                           scale, s);
                }
            }
        }
        free(Kc);
        free(Vc);
        free(s);
        free(qv);
    }
    return status;
}

int pa_oracle_prefill(double *out, const void *q, const void *k_cache, const void *v_cache, int dtype,
                      const int32_t *block_tables, int max_blocks_per_seq, const int32_t *cu_q_lens,
                      const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads,
                      int head_dim, int block_size, long num_blocks, double scale,
                      const int32_t *rows, long n_rows, int num_threads)
{
    return prefill_impl(out, q, dtype, k_cache, v_cache, dtype, 1.0, 1.0, block_tables, max_blocks_per_seq,
                        cu_q_lens, context_lens, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                        num_blocks, scale, rows, n_rows, num_threads);
}

/*
 * Prefill chunk over FP8 E4M3 caches: K = e4m3(code) * k_scale, V =
 * e4m3(code) * v_scale, q and out as q_dtype. Otherwise identical to
 * pa_oracle_prefill.
 */
int pa_oracle_prefill_fp8(double *out, const void *q, int q_dtype, const uint8_t *k_cache,
                          const uint8_t *v_cache, double k_scale, double v_scale, const int32_t *block_tables,
                          int max_blocks_per_seq, const int32_t *cu_q_lens, const int32_t *context_lens,
                          int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                          long num_blocks, double scale, const int32_t *rows, long n_rows, int num_threads)
{
    return prefill_impl(out, q, q_dtype, k_cache, v_cache, ORACLE_FP8_E4M3, k_scale, v_scale, block_tables,
                        max_blocks_per_seq, cu_q_lens, context_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                        block_size, num_blocks, scale, rows, n_rows, num_threads);
}

/*
 * Cache write: for each token t with slot_mapping[t] >= 0, copy token_bytes
 * of k[t] into k_cache at slot_mapping[t] * token_bytes, and the same for v.
 * A token row is [kv_heads][head_dim] elements. Every other byte is left
 * as it was. Returns the number of tokens written, or -1 (nothing written)
 * if any slot is >= num_slots.
 */
long pa_oracle_reshape_and_cache(const void *k, const void *v, void *k_cache, void *v_cache,
                                 const int64_t *slot_mapping, long num_tokens, long num_slots,
                                 long token_bytes)
{
    for (long t = 0; t < num_tokens; ++t)
        if (slot_mapping[t] >= num_slots)
            return -1;
    long written = 0;
    for (long t = 0; t < num_tokens; ++t) {
        long s = slot_mapping[t];
        if (s < 0)
            continue;
        if (g_mutation == MUT_WRITE_NEXT && s + 1 < num_slots)
            s += 1;
        memcpy((char *)k_cache + s * token_bytes, (const char *)k + t * token_bytes, (size_t)token_bytes);
        memcpy((char *)v_cache + s * token_bytes, (const char *)v + t * token_bytes, (size_t)token_bytes);
        ++written;
    }
    return written;
}

/*
 * Block copies. The pages share identical prefixes by pointing several tables
 * at the same physical blocks and copy a block before it is written
 * (copy-on-write: "vLLM — PagedAttention and Continuous Batching" §2.3,
 * "vLLM and PagedAttention" §2 "The PagedAttention Solution", "How vLLM
 * Works?" §03). Preemption moves a request's blocks out to host memory and
 * back ("vLLM and PagedAttention" §3; "How vLLM Works?" §04).
 *
 * pa_oracle_copy_blocks: for each pair i in order, block pairs[2i+1] of both
 * pools becomes a byte copy of block pairs[2i]. block_bytes is one block of
 * one pool (block_size * kv_heads * head_dim * elem). Returns 0, or -1 (and
 * copies nothing) if an index is outside [0, num_blocks).
 */
int pa_oracle_copy_blocks(void *k_cache, void *v_cache, const int64_t *pairs, long num_pairs, long num_blocks,
                          long block_bytes)
{
    for (long i = 0; i < 2 * num_pairs; ++i)
        if (pairs[i] < 0 || pairs[i] >= num_blocks)
            return -1;
    for (long i = 0; i < num_pairs; ++i) {
        long src = pairs[2 * i], dst = pairs[2 * i + 1];
        memmove((char *)k_cache + dst * block_bytes, (const char *)k_cache + src * block_bytes, (size_t)block_bytes);
        memmove((char *)v_cache + dst * block_bytes, (const char *)v_cache + src * block_bytes, (size_t)block_bytes);
    }
    return 0;
}

/*
 * pa_oracle_swap_blocks: for each pair i, block pairs[2i+1] of dst becomes a
 * byte copy of block pairs[2i] of src (one pool; call once for K and once for
 * V). src and dst may hold different numbers of blocks. Returns 0 or -1.
 */
int pa_oracle_swap_blocks(void *dst, const void *src, const int64_t *pairs, long num_pairs, long src_blocks,
                          long dst_blocks, long block_bytes)
{
    for (long i = 0; i < num_pairs; ++i)
        if (pairs[2 * i] < 0 || pairs[2 * i] >= src_blocks || pairs[2 * i + 1] < 0 || pairs[2 * i + 1] >= dst_blocks)
            return -1;
    for (long i = 0; i < num_pairs; ++i)
        memcpy((char *)dst + pairs[2 * i + 1] * block_bytes, (const char *)src + pairs[2 * i] * block_bytes,
               (size_t)block_bytes);
    return 0;
}

/*
 * FP8 cache write: the new tokens' K/V rows (bf16 bits) are quantized to E4M3
 * with the same fp32 steps the kernel takes: x -> fp32, times inv_scale in
 * fp32 (one IEEE multiply), then E4M3 rounding. Dequantized value =
 * e4m3(code) * scale with scale = 1 / inv_scale. Returns tokens written or -1.
 */
long pa_oracle_reshape_and_cache_fp8(const uint16_t *k, const uint16_t *v, uint8_t *k_cache, uint8_t *v_cache,
                                     const int64_t *slot_mapping, long num_tokens, long num_slots, long row_elems,
                                     float k_inv_scale, float v_inv_scale)
{
    for (long t = 0; t < num_tokens; ++t)
        if (slot_mapping[t] >= num_slots)
            return -1;
    long written = 0;
    for (long t = 0; t < num_tokens; ++t) {
        long s = slot_mapping[t];
        if (s < 0)
            continue;
        for (long i = 0; i < row_elems; ++i) {
            uint32_t ku = (uint32_t)k[t * row_elems + i] << 16, vu = (uint32_t)v[t * row_elems + i] << 16;
            float kf, vf;
            memcpy(&kf, &ku, 4);
            memcpy(&vf, &vu, 4);
            volatile float kq = kf * k_inv_scale, vq = vf * v_inv_scale; /* fp32 products */
            k_cache[s * row_elems + i] = pa_oracle_e4m3_encode(kq);
            v_cache[s * row_elems + i] = pa_oracle_e4m3_encode(vq);
        }
        ++written;
    }
    return written;
}

/*
 * Decode over an FP8 E4M3 cache: K = e4m3(code) * k_scale, V = e4m3(code) *
 * v_scale, q and out as q_dtype. Otherwise identical to pa_oracle_decode.
 */
int pa_oracle_decode_fp8(double *out, const void *q, int q_dtype, const uint8_t *k_cache, const uint8_t *v_cache,
                         double k_scale, double v_scale, const int32_t *block_tables, int max_blocks_per_seq,
                         const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                         int block_size, long num_blocks, double scale, int num_threads)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0)
        return -2;
    int nt = set_threads(num_threads);
    int status = 0;
    long units = (long)num_seqs * num_kv_heads;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (long u = 0; u < units; ++u) {
        int b = (int)(u / num_kv_heads), hk = (int)(u % num_kv_heads);
        long c = context_lens[b];
        double *Kc = malloc(sizeof(double) * (size_t)(c > 0 ? c : 1) * head_dim);
        double *Vc = malloc(sizeof(double) * (size_t)(c > 0 ? c : 1) * head_dim);
        double *s = malloc(sizeof(double) * (size_t)(c > 0 ? c : 1));
        double *qv = malloc(sizeof(double) * (size_t)head_dim);
        int rc = (c < 0) ? -2 : pa_oracle_gather(Kc, Vc, k_cache, v_cache, ORACLE_FP8_E4M3, block_tables,
                                                  max_blocks_per_seq, b, c, num_kv_heads, hk, head_dim,
                                                  block_size, num_blocks);
        if (rc) {
#pragma omp critical
            status = rc;
        } else {
            for (long i = 0; i < c * head_dim; ++i) {
                Kc[i] *= k_scale;
                Vc[i] *= v_scale;
            }
            for (int h = 0; h < num_heads; ++h) {
                if (kv_head_of(h, num_heads, num_kv_heads) != hk)
                    continue;
                long qbase = ((long)b * num_heads + h) * head_dim;
                for (int d = 0; d < head_dim; ++d)
                    qv[d] = load_elem(q, qbase + d, q_dtype);
                attend(out + qbase, qv, Kc, Vc, readable_tokens(c, block_size), head_dim, scale, s);
            }
        }
        free(Kc);
        free(Vc);
        free(s);
        free(qv);
    }
    return status;
}
