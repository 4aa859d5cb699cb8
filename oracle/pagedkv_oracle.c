/*
 * ORACLE -- test infrastructure, not product code.
 *
 * A plain, slow, obviously-correct CPU statement of what the paged KV-cache
 * decode path computes, in float64.  Only the test suite, the smoke check and
 * the benchmark's CPU-baseline leg may call it; the CUDA library never links
 * or calls it, and this file shares no code, header or table with the CUDA
 * sources.
 *
 * Sources (web pages on PagedAttention):
 *   [UL]  Ultralytics glossary "PagedAttention" (Japanese), sections
 *         "How paging works" (worked PyTorch example: scatter of keys into a
 *         shared block pool through a block table, and the gather back),
 *         "Sharing blocks across sequences" (ref counts, copy-on-write),
 *         "Related methods" (FlashAttention-style tiling, GQA, FP8 cache).
 *   [WP]  Wikipedia "PagedAttention" (mirror), section "Mathematical
 *         formulation": token-form causal attention a_ij / o_i and the
 *         block form A_ij / o_i over ceil(i/B) blocks, which the page states
 *         preserves the causal attention result.
 *   [PT]  "vLLM and PagedAttention: virtual memory for LLM inference"
 *         (podcast transcript): copy of the partially filled shared block on
 *         write, full shared blocks stay shared.
 *   [PT]  (same transcript, opening paragraph): inference splits into the
 *         prefill of the prompt, whose tokens are all known at once and map
 *         onto large matrix products, and the token-by-token decode.
 *   [HJ]  "Paged Attention" study notes (huajishe.fun), section on
 *         points to watch: the first forward pass of a new request (prefill)
 *         needs its own handling.
 *   [OCP] OCP 8-bit Floating Point Specification (OFP8), E4M3 encoding:
 *         bias 7, no infinities, S.1111.111 is NaN, max finite 448,
 *         subnormals m * 2^-9.  The pages only say "8-bit"; the choice of
 *         E4M3 is a reading of them.
 *
 * Because the blockwise method reaches exactly the plain causal-attention
 * result ([WP]), the decode oracle below is that plain definition (gather
 * through the table, then textbook two-pass softmax), not the blockwise
 * algorithm.  Readings where the pages are silent:
 *   - the query of a decode step is the last cached token, so attention
 *     covers positions 0..L-1 of a sequence whose context length is L;
 *   - only tokens t < L count: unused slots of the last block are masked;
 *   - query head h uses KV head h / (H / Hkv) (contiguous GQA groups);
 *   - pool layout [num_blocks][num_kv_heads][block_size][head_dim];
 *   - FP8 dequantisation is decode_e4m3(byte) * scale, quantisation is
 *     round-to-nearest-even with saturation of float32(x) / scale, the
 *     division done in IEEE float32.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F16 = 0, ORC_BF16 = 1, ORC_E4M3 = 2 };

enum {
    ORC_OK = 0,
    ORC_BAD_ARG = 1,      /* a size or dtype outside what the oracle handles   */
    ORC_BAD_BLOCK = 2,    /* a block-table entry outside [0, num_blocks)        */
    ORC_BAD_SLOT = 3,     /* a slot beyond num_blocks * block_size              */
    ORC_BAD_LEN = 4       /* a context length beyond the table's capacity       */
};

/* ---------------------------------------------------------------------- */
/* Number formats, decoded from their definitions.                        */
/* ---------------------------------------------------------------------- */

/* IEEE 754 binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double orc_f16_to_f64(uint16_t h)
{
    int sign = h >> 15, e = (h >> 10) & 0x1f, m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* 0.m * 2^-14 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);     /* 1.m * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16: 1 sign, 8 exponent (bias 127), 7 fraction bits. */
double orc_bf16_to_f64(uint16_t h)
{
    int sign = h >> 15, e = (h >> 7) & 0xff, m = h & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)m, -133);                /* 0.m * 2^-126 */
    else if (e == 255)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + m), e - 134);     /* 1.m * 2^(e-127) */
    return sign ? -v : v;
}

/* OCP E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; S.1111.111 = NaN. */
double orc_e4m3_to_f64(uint8_t b)
{
    int sign = b >> 7, e = (b >> 3) & 0xf, m = b & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);                  /* 0.mmm * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10);        /* 1.mmm * 2^(e-7) */
    return sign ? -v : v;
}

/* float32 -> E4M3, round to nearest even, saturating to +-448; NaN -> S.1111.111. */
uint8_t orc_f32_to_e4m3(float x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs((double)x);
    if (isnan(x))
        return sign | 0x7f;
    if (a >= 448.0)
        return sign | 0x7e;                          /* saturate */
    /* quantum of the E4M3 grid at a: 2^-9 below the smallest normal 2^-6,
     * else 2^(floor(log2 a) - 3). */
    double quantum;
    if (a < ldexp(1.0, -6)) {
        quantum = ldexp(1.0, -9);
    } else {
        int ex;
        frexp(a, &ex);                               /* a = f * 2^ex, f in [0.5,1) */
        quantum = ldexp(1.0, (ex - 1) - 3);
    }
    double q = a / quantum;                          /* exact: power-of-two scaling */
    double r = nearbyint(q);                         /* default mode: ties to even */
    double v = r * quantum;
    if (v > 448.0)
        v = 448.0;
    if (v == 0.0)
        return sign;
    if (v < ldexp(1.0, -6))
        return sign | (uint8_t)(v / ldexp(1.0, -9)); /* subnormal: mantissa only */
    int ex;
    double f = frexp(v, &ex);                        /* v = f * 2^ex */
    int unb = ex - 1;                                /* v in [2^unb, 2^(unb+1)) */
    int mant = (int)(f * 16.0) - 8;                  /* (v / 2^unb) = 1 + mant/8 */
    return sign | (uint8_t)(((unb + 7) << 3) | mant);
}

/*
 * Every 16-bit pattern's value, filled once from the decoders above: the
 * attention loops read each cached element many times, and a table lookup
 * gives the same float64 value as calling the decoder again, only faster.
 */
static double f16_value[65536], bf16_value[65536];
static pthread_once_t value_tables_once = PTHREAD_ONCE_INIT;

static void fill_value_tables(void)
{
    for (uint32_t h = 0; h < 65536; ++h) {
        f16_value[h] = orc_f16_to_f64((uint16_t)h);
        bf16_value[h] = orc_bf16_to_f64((uint16_t)h);
    }
}

static double load_elem(const void* base, size_t idx, int dtype, double scale)
{
    switch (dtype) {
    case ORC_F16:  return f16_value[((const uint16_t*)base)[idx]];
    case ORC_BF16: return bf16_value[((const uint16_t*)base)[idx]];
    default:       return orc_e4m3_to_f64(((const uint8_t*)base)[idx]) * scale;
    }
}

static size_t elem_bytes(int dtype) { return dtype == ORC_E4M3 ? 1 : 2; }

/* ---------------------------------------------------------------------- */
/* Decode attention ([WP] "Mathematical formulation", token form).         */
/* ---------------------------------------------------------------------- */

/*
 * out[s][h][:] = sum_{t<L_s} softmax_t(scale * q[s][h] . k_t) v_t  in float64,
 * where k_t, v_t are read through the block table as in [UL]'s gather:
 *   pid = block_tables[s][t / B], off = t % B, k_t = k_pool[pid][h/G][off][:].
 * Sequences with L_s = 0 give a zero output.
 */
int orc_paged_attn_decode(double* out, const void* q, int q_dtype,
                          const void* k_pool, const void* v_pool, int kv_dtype,
                          double k_scale, double v_scale,
                          const int32_t* block_tables, int max_blocks_per_seq,
                          const int32_t* context_lens, int num_seqs, int num_heads,
                          int num_kv_heads, int head_dim, int block_size,
                          int num_blocks, double scale, int num_threads)
{
    pthread_once(&value_tables_once, fill_value_tables);
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_blocks <= 0 || num_heads % num_kv_heads != 0 ||
        (q_dtype != ORC_F16 && q_dtype != ORC_BF16) ||
        (kv_dtype != ORC_F16 && kv_dtype != ORC_BF16 && kv_dtype != ORC_E4M3))
        return ORC_BAD_ARG;
    const int G = num_heads / num_kv_heads;
    const double ks = kv_dtype == ORC_E4M3 ? k_scale : 1.0;
    const double vs = kv_dtype == ORC_E4M3 ? v_scale : 1.0;

    /* validate every table entry that the definition reads */
    for (int s = 0; s < num_seqs; ++s) {
        int L = context_lens[s];
        if (L < 0 || L > (long)max_blocks_per_seq * block_size)
            return ORC_BAD_LEN;
        for (int j = 0; j < (L + block_size - 1) / block_size; ++j) {
            int pid = block_tables[(size_t)s * max_blocks_per_seq + j];
            if (pid < 0 || pid >= num_blocks)
                return ORC_BAD_BLOCK;
        }
    }

#ifdef _OPENMP
    if (num_threads > 0)
        omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
    const long units = (long)num_seqs * num_heads;
#pragma omp parallel
    {
        int maxL = 0;
        for (int s = 0; s < num_seqs; ++s)
            if (context_lens[s] > maxL) maxL = context_lens[s];
        double* x = (double*)malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
        double* qv = (double*)malloc(sizeof(double) * (size_t)head_dim);
#pragma omp for schedule(dynamic, 1)
        for (long u = 0; u < units; ++u) {
            const int s = (int)(u / num_heads), h = (int)(u % num_heads);
            const int kvh = h / G;
            const int L = context_lens[s];
            double* o = out + (size_t)u * head_dim;
            for (int d = 0; d < head_dim; ++d) {
                o[d] = 0.0;
                qv[d] = load_elem(q, (size_t)u * head_dim + d, q_dtype, 1.0);
            }
            if (L == 0)
                continue;
            /* pass 1: scores and their maximum */
            double m = -INFINITY;
            for (int t = 0; t < L; ++t) {
                int pid = block_tables[(size_t)s * max_blocks_per_seq + t / block_size];
                size_t row = (((size_t)pid * num_kv_heads + kvh) * block_size + t % block_size) * head_dim;
                double dot = 0.0;
                for (int d = 0; d < head_dim; ++d)
                    dot += qv[d] * load_elem(k_pool, row + d, kv_dtype, ks);
                x[t] = scale * dot;
                if (x[t] > m) m = x[t];
            }
            /* pass 2: p_t = exp(x_t - m), l = sum p_t, o = sum p_t v_t / l */
            double l = 0.0;
            for (int t = 0; t < L; ++t) {
                double p = exp(x[t] - m);
                l += p;
                int pid = block_tables[(size_t)s * max_blocks_per_seq + t / block_size];
                size_t row = (((size_t)pid * num_kv_heads + kvh) * block_size + t % block_size) * head_dim;
                for (int d = 0; d < head_dim; ++d)
                    o[d] += p * load_elem(v_pool, row + d, kv_dtype, vs);
            }
            for (int d = 0; d < head_dim; ++d)
                o[d] /= l;
        }
        free(x);
        free(qv);
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------- */
/* Chunked prefill ([WP] token form for every query position of a chunk;   */
/* [PT] prefill; [HJ] prefill handling).                                    */
/* ---------------------------------------------------------------------- */

/*
 * Sequence s holds L_s = context_lens[s] tokens in the cache; its last
 * C_s = query_start[s+1] - query_start[s] tokens are the chunk being
 * prefilled (their K/V already scattered into the pool, as for decode).
 * Query row r = query_start[s] + j (j < C_s) is token position
 * p = L_s - C_s + j and attends causally to positions 0..p:
 *   out[r][h][:] = sum_{t<=p} softmax_t(scale * q[r][h] . k_t) v_t,
 * with k_t, v_t read through the block table as in decode.  Decode is the
 * case C_s = 1.  q is [num_tokens][H][D] with num_tokens = query_start[S].
 */
int orc_paged_attn_prefill(double* out, const void* q, int q_dtype,
                           const void* k_pool, const void* v_pool, int kv_dtype,
                           double k_scale, double v_scale,
                           const int32_t* block_tables, int max_blocks_per_seq,
                           const int32_t* context_lens, const int32_t* query_start,
                           int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                           int block_size, int num_blocks, double scale, int num_threads)
{
    pthread_once(&value_tables_once, fill_value_tables);
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_blocks <= 0 || num_heads % num_kv_heads != 0 ||
        (q_dtype != ORC_F16 && q_dtype != ORC_BF16) ||
        (kv_dtype != ORC_F16 && kv_dtype != ORC_BF16 && kv_dtype != ORC_E4M3) ||
        query_start[0] != 0)
        return ORC_BAD_ARG;
    const int G = num_heads / num_kv_heads;
    const double ks = kv_dtype == ORC_E4M3 ? k_scale : 1.0;
    const double vs = kv_dtype == ORC_E4M3 ? v_scale : 1.0;
    for (int s = 0; s < num_seqs; ++s) {
        const int L = context_lens[s], C = query_start[s + 1] - query_start[s];
        if (C < 0 || C > L)
            return ORC_BAD_ARG;
        if (L > (long)max_blocks_per_seq * block_size)
            return ORC_BAD_LEN;
        for (int j = 0; j < (L + block_size - 1) / block_size; ++j) {
            int pid = block_tables[(size_t)s * max_blocks_per_seq + j];
            if (pid < 0 || pid >= num_blocks)
                return ORC_BAD_BLOCK;
        }
    }
    const long rows = query_start[num_seqs];
#ifdef _OPENMP
    if (num_threads > 0)
        omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel
    {
        int maxL = 1;
        for (int s = 0; s < num_seqs; ++s)
            if (context_lens[s] > maxL) maxL = context_lens[s];
        double* x = (double*)malloc(sizeof(double) * (size_t)maxL);
        double* qv = (double*)malloc(sizeof(double) * (size_t)head_dim);
#pragma omp for schedule(dynamic, 1)
        for (long u = 0; u < rows * num_heads; ++u) {
            const long r = u / num_heads;
            const int h = (int)(u % num_heads), kvh = h / G;
            int s = 0;
            while (query_start[s + 1] <= r) ++s;          /* the sequence row r belongs to */
            const int L = context_lens[s];
            const int C = query_start[s + 1] - query_start[s];
            const int p = L - C + (int)(r - query_start[s]);   /* its token position */
            double* o = out + (size_t)u * head_dim;
            for (int d = 0; d < head_dim; ++d) {
                o[d] = 0.0;
                qv[d] = load_elem(q, (size_t)u * head_dim + d, q_dtype, 1.0);
            }
            double m = -INFINITY;
            for (int t = 0; t <= p; ++t) {
                int pid = block_tables[(size_t)s * max_blocks_per_seq + t / block_size];
                size_t krow = (((size_t)pid * num_kv_heads + kvh) * block_size + t % block_size) * head_dim;
                double dot = 0.0;
                for (int d = 0; d < head_dim; ++d)
                    dot += qv[d] * load_elem(k_pool, krow + d, kv_dtype, ks);
                x[t] = scale * dot;
                if (x[t] > m) m = x[t];
            }
            double l = 0.0;
            for (int t = 0; t <= p; ++t) {
                double w = exp(x[t] - m);
                l += w;
                int pid = block_tables[(size_t)s * max_blocks_per_seq + t / block_size];
                size_t vrow = (((size_t)pid * num_kv_heads + kvh) * block_size + t % block_size) * head_dim;
                for (int d = 0; d < head_dim; ++d)
                    o[d] += w * load_elem(v_pool, vrow + d, kv_dtype, vs);
            }
            for (int d = 0; d < head_dim; ++d)
                o[d] /= l;
        }
        free(x);
        free(qv);
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------- */
/* Scatter of new tokens into the pool ([UL] "How paging works":           */
/*   key_pool[block_table[pos // B], pos % B] = key).                      */
/* ---------------------------------------------------------------------- */

/*
 * For each token t and KV head h with slot = slot_mapping[t] >= 0:
 *   pool[slot / B][h][slot % B][:] = k[t][h][:]   (same for v),
 * copied bit for bit when the pool has the input's 16-bit type, or stored as
 * e4m3(float32(x) / scale) for an E4M3 pool.  Negative slots are skipped.
 */
int orc_reshape_and_cache(const void* k, const void* v, int in_dtype,
                          void* k_pool, void* v_pool, int kv_dtype,
                          float k_scale, float v_scale,
                          const int64_t* slot_mapping, int num_tokens,
                          int num_kv_heads, int head_dim, int block_size, int num_blocks)
{
    pthread_once(&value_tables_once, fill_value_tables);
    if ((in_dtype != ORC_F16 && in_dtype != ORC_BF16) ||
        (kv_dtype != in_dtype && kv_dtype != ORC_E4M3) || num_tokens < 0 ||
        num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return ORC_BAD_ARG;
    for (int t = 0; t < num_tokens; ++t)
        if (slot_mapping[t] >= (int64_t)num_blocks * block_size)
            return ORC_BAD_SLOT;
    for (int t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        int64_t blk = slot / block_size, off = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            size_t src = ((size_t)t * num_kv_heads + h) * head_dim;
            size_t dst = (((size_t)blk * num_kv_heads + h) * block_size + off) * head_dim;
            for (int d = 0; d < head_dim; ++d) {
                if (kv_dtype == in_dtype) {
                    ((uint16_t*)k_pool)[dst + d] = ((const uint16_t*)k)[src + d];
                    ((uint16_t*)v_pool)[dst + d] = ((const uint16_t*)v)[src + d];
                } else {
                    /* the 16-bit value is exact in float32; divide in float32 */
                    float kx = (float)load_elem(k, src + d, in_dtype, 1.0);
                    float vx = (float)load_elem(v, src + d, in_dtype, 1.0);
                    volatile float kq = kx / k_scale;
                    volatile float vq = vx / v_scale;
                    ((uint8_t*)k_pool)[dst + d] = orc_f32_to_e4m3(kq);
                    ((uint8_t*)v_pool)[dst + d] = orc_f32_to_e4m3(vq);
                }
            }
        }
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------- */
/* Block-granular copy-on-write ([UL] "Sharing blocks across sequences";   */
/* [PT]: only the partially filled shared block is copied).                */
/* ---------------------------------------------------------------------- */

/* pool[dst] := pool[src] for every (src, dst) pair, K and V, in pair order. */
int orc_copy_blocks(void* k_pool, void* v_pool, size_t block_bytes,
                    const int64_t* pairs, int num_pairs, int num_blocks)
{
    if (num_pairs < 0 || num_blocks <= 0 || block_bytes == 0)
        return ORC_BAD_ARG;
    for (int i = 0; i < num_pairs; ++i) {
        int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
        if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks)
            return ORC_BAD_BLOCK;
    }
    for (int i = 0; i < num_pairs; ++i) {
        int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
        memmove((char*)k_pool + (size_t)d * block_bytes, (char*)k_pool + (size_t)s * block_bytes, block_bytes);
        memmove((char*)v_pool + (size_t)d * block_bytes, (char*)v_pool + (size_t)s * block_bytes, block_bytes);
    }
    return ORC_OK;
}

/*
 * Swap between two pools ([PT], on preemption: a group's KV data moves to CPU
 * memory and is brought back later): for each pair (s, d),
 *   dst_k[d] := src_k[s] and dst_v[d] := src_v[s], whole blocks, bit for bit.
 */
int orc_swap_blocks(const void* src_k, const void* src_v, int src_blocks, void* dst_k, void* dst_v,
                    int dst_blocks, size_t block_bytes, const int64_t* pairs, int num_pairs)
{
    if (num_pairs < 0 || src_blocks <= 0 || dst_blocks <= 0 || block_bytes == 0)
        return ORC_BAD_ARG;
    for (int i = 0; i < num_pairs; ++i) {
        int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
        if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks)
            return ORC_BAD_BLOCK;
    }
    for (int i = 0; i < num_pairs; ++i) {
        int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
        memcpy((char*)dst_k + (size_t)d * block_bytes, (const char*)src_k + (size_t)s * block_bytes, block_bytes);
        memcpy((char*)dst_v + (size_t)d * block_bytes, (const char*)src_v + (size_t)s * block_bytes, block_bytes);
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------- */
/* Gather through the table ([UL]: pool[block_table].reshape(-1, d)[:len]) */
/* ---------------------------------------------------------------------- */

/* out[t][:] = pool[table[t / B]][kvh][t % B][:] for t < len, raw bytes. */
int orc_gather(void* out, const void* pool, int kv_dtype, const int32_t* table,
               int table_len, int len, int num_kv_heads, int kvh, int head_dim,
               int block_size, int num_blocks)
{
    if (len < 0 || len > (long)table_len * block_size || kvh < 0 || kvh >= num_kv_heads)
        return ORC_BAD_ARG;
    size_t eb = elem_bytes(kv_dtype);
    for (int t = 0; t < len; ++t) {
        int pid = table[t / block_size];
        if (pid < 0 || pid >= num_blocks)
            return ORC_BAD_BLOCK;
        size_t row = (((size_t)pid * num_kv_heads + kvh) * block_size + t % block_size) * head_dim;
        memcpy((char*)out + (size_t)t * head_dim * eb, (const char*)pool + row * eb, head_dim * eb);
    }
    return ORC_OK;
}

/* Element-wise decoders over arrays, for the tests' exhaustive checks. */
void orc_decode_array(double* out, const void* in, int dtype, size_t n)
{
    pthread_once(&value_tables_once, fill_value_tables);
    for (size_t i = 0; i < n; ++i)
        out[i] = load_elem(in, i, dtype, 1.0);
}

void orc_encode_e4m3_array(uint8_t* out, const float* in, size_t n)
{
    for (size_t i = 0; i < n; ++i)
        out[i] = orc_f32_to_e4m3(in[i]);
}
