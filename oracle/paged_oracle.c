/*
 * Paged-KV oracle: plain, slow, obviously correct CPU reference (fp64).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library.
 *
 * Sources followed (page title, then the section on that page):
 *   [T1] "LLM推理优化实战：从KV Cache到Speculative Decoding，把延迟打下来"
 *   [T2] "大模型推理加速：从 KV Cache 到投机采样的工程实践"
 *   [T3] "LLM 推理优化：KV Cache、PagedAttention 与量化"
 *   [T4] "大模型推理加速与显存黑科技 (Inference Acceleration & KV Cache)"
 *
 * What is computed, and where the pages fix it:
 *   - attention = softmax(Q K^T * scale) V, exactly, per query row
 *     ([T4] §2 "KV Cache：空间换时间的经典范式", the Attention(Q,K,V) formula;
 *      scale = 1/sqrt(d_k) there, and d_head**-0.5 in [T1] §"KV Cache：推理加速的
 *      第一板斧"; the caller passes the scale).
 *   - the KV cache of a sequence is cut into fixed-size blocks; logical block b
 *     holds tokens [b*bs, b*bs + bs) and a per-sequence block table maps it to a
 *     physical block ([T3] §2.2 "解法：借鉴 OS 虚拟内存"; [T4] §3.2, the
 *     logical -> block table -> physical figure with 16-token blocks).
 *   - grouped-query attention: query heads are split into groups and every
 *     group shares one KV head ([T2] §"主流优化策略", MQA/GQA).  Contiguous
 *     groups are used: query head h reads KV head h / (Hq / Hkv).
 *   - speculative verify: the target model scores the draft tokens in one
 *     forward pass over prompt + drafts ([T1] §"Speculative Decoding：用草稿
 *     模型加速"; [T3] §6.2).  Read causally: row j of a q_len window sees
 *     keys 0 .. L - q_len + j, where L counts the drafts.
 *   - appending a token writes its K/V into the slot the host reserved; a
 *     copy-on-write fork copies a whole physical block ([T3] §2.3 (2)
 *     "Copy-on-Write").
 *   - KV bytes = 2 x layers x heads x head_dim x seq_len x batch x dtype_size
 *     ([T2] §"KV Cache的内存挑战"; [T4] §2.1 with the two factors of 2 spelled
 *     out; worked example in [T1] §"KV Cache：推理加速的第一板斧": LLaMA-2 70B,
 *     80 layers, 64 heads, 128 dims -> about 2.5 GB per 1K tokens).
 *
 * Layouts (the pages fix none; these are the plainest reading, shared with the
 * CUDA library only by their written definition):
 *   q            fp16 [B][q_len][Hq][D]
 *   k/v pool     fp16 [num_blocks][Hkv][bs][D]
 *   block_tables int32 [B][max_blocks_per_seq]
 *   context_lens int32 [B]
 *   out          fp64 [B][q_len][Hq][D]
 * fp16 values travel as their raw 16-bit patterns (uint16_t) and are decoded
 * here from the IEEE 754 binary16 definition.
 *
 * Pins: every function here is checked against something other than itself
 * (closed forms, a textbook attention routine on a contiguous cache, brute
 * force, the worked memory example) by the CPU tests; none is unpinned.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_TABLE 2

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * exponent 0 -> subnormal (fraction * 2^-24); exponent 31 -> inf / nan. */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double v;
    if (expo == 0) {
        v = ldexp((double)frac, -24);
    } else if (expo == 31) {
        v = frac ? NAN : INFINITY;
    } else {
        v = ldexp((double)(frac | 0x400), expo - 25);
    }
    return sign ? -v : v;
}

/* Number of threads the OpenMP loops below will use. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* KV cache bytes, the pages' formula taken literally. */
uint64_t oracle_kv_cache_bytes(uint64_t layers, uint64_t heads, uint64_t head_dim,
                               uint64_t seq_len, uint64_t batch, uint64_t dtype_bytes)
{
    return 2ull * layers * heads * head_dim * seq_len * batch * dtype_bytes;
}

/* Bytes of one layer's K pool plus V pool: the same formula with the pool's
 * capacity (num_blocks * block_size tokens) in place of seq_len * batch and
 * the KV heads in place of heads (under MQA/GQA only the KV heads are cached). */
uint64_t oracle_pool_bytes_per_layer(uint64_t num_blocks, uint64_t block_size,
                                     uint64_t num_kv_heads, uint64_t head_dim,
                                     uint64_t dtype_bytes)
{
    return oracle_kv_cache_bytes(1, num_kv_heads, head_dim, num_blocks * block_size, 1,
                                 dtype_bytes);
}

/* Address of element [p][kvh][o][0] of a pool. */
static size_t pool_row(int64_t p, int32_t kvh, int32_t o, int32_t Hkv, int32_t bs, int32_t D)
{
    return (((size_t)p * (size_t)Hkv + (size_t)kvh) * (size_t)bs + (size_t)o) * (size_t)D;
}

/*
 * Exact attention over paged K/V for every (sequence, window row, query head).
 *
 * For sequence s, window row j (0 <= j < q_len) and query head h:
 *   kvh   = h / (Hq / Hkv)
 *   L     = context_lens[s]; last = L - q_len + j  (decode: q_len = 1, last = L-1)
 *   for t = 0 .. last:  p = block_tables[s][t / bs], o = t % bs
 *                       K_t = k_pool[p][kvh][o][:],  V_t = v_pool[p][kvh][o][:]
 *                       s_t = scale * sum_d q[s][j][h][d] * K_t[d]
 *   M = max_t s_t,  w_t = exp(s_t - M),  Z = sum_t w_t
 *   out[s][j][h][:] = sum_t w_t V_t / Z
 * A row that sees no key (last < 0) is all zeros.
 * K is read from an fp16 pool (k16), or from an 8-bit code pool (k8) as
 * code * k_scales[kvh][d] (see the quantised pool below).
 * Returns ORACLE_ERR_TABLE if a table entry that is read lies outside
 * [0, num_blocks), ORACLE_ERR_ARG on bad sizes.
 */
static int attention_rows(const uint16_t* q, const uint16_t* k16, const int8_t* k8,
                          const float* k_scales, const uint16_t* v_pool,
                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                          const int32_t* context_lens, int32_t B, int32_t q_len, int32_t Hq,
                          int32_t Hkv, int32_t D, int32_t bs, int32_t num_blocks, double scale,
                          double* out)
{
    if (B < 0 || q_len < 1 || Hq < 1 || Hkv < 1 || D < 1 || bs < 1 || Hq % Hkv != 0)
        return ORACLE_ERR_ARG;
    for (int32_t s = 0; s < B; ++s) {
        int32_t L = context_lens[s];
        if (L < 0 || (int64_t)(L + bs - 1) / bs > max_blocks_per_seq) return ORACLE_ERR_ARG;
        for (int32_t b = 0; b < (L + bs - 1) / bs; ++b) {
            int32_t p = block_tables[(size_t)s * max_blocks_per_seq + b];
            if (p < 0 || p >= num_blocks) return ORACLE_ERR_TABLE;
        }
    }
    const int32_t group = Hq / Hkv;
    const int64_t rows = (int64_t)B * q_len * Hq;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        const int32_t h = (int32_t)(r % Hq);
        const int32_t j = (int32_t)((r / Hq) % q_len);
        const int32_t s = (int32_t)(r / ((int64_t)Hq * q_len));
        const int32_t kvh = h / group;
        const int32_t L = context_lens[s];
        const int32_t last = L - q_len + j;
        const uint16_t* qrow = q + (size_t)r * D;
        double* orow = out + (size_t)r * D;
        for (int32_t d = 0; d < D; ++d) orow[d] = 0.0;
        if (last < 0) continue;
        const int32_t n = last + 1;

        double* qd = (double*)malloc(sizeof(double) * (size_t)D);
        double* sc = (double*)malloc(sizeof(double) * (size_t)n);
        for (int32_t d = 0; d < D; ++d) qd[d] = oracle_half_to_double(qrow[d]);

        /* scores */
        double M = -INFINITY;
        for (int32_t t = 0; t < n; ++t) {
            int32_t p = block_tables[(size_t)s * max_blocks_per_seq + t / bs];
            const size_t row = pool_row(p, kvh, t % bs, Hkv, bs, D);
            double dot = 0.0;
            for (int32_t d = 0; d < D; ++d) {
                const double kd = k8 ? (double)k8[row + d] * (double)k_scales[(size_t)kvh * D + d]
                                     : oracle_half_to_double(k16[row + d]);
                dot += qd[d] * kd;
            }
            sc[t] = scale * dot;
            if (sc[t] > M) M = sc[t];
        }
        /* softmax weights and the weighted sum of values */
        double Z = 0.0;
        for (int32_t t = 0; t < n; ++t) {
            double w = exp(sc[t] - M);
            sc[t] = w;
            Z += w;
        }
        for (int32_t t = 0; t < n; ++t) {
            int32_t p = block_tables[(size_t)s * max_blocks_per_seq + t / bs];
            const uint16_t* vrow = v_pool + pool_row(p, kvh, t % bs, Hkv, bs, D);
            for (int32_t d = 0; d < D; ++d) orow[d] += sc[t] * oracle_half_to_double(vrow[d]);
        }
        for (int32_t d = 0; d < D; ++d) orow[d] /= Z;
        free(qd);
        free(sc);
    }
    return ORACLE_OK;
}

int oracle_paged_attention(const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                           const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* context_lens, int32_t B, int32_t q_len, int32_t Hq,
                           int32_t Hkv, int32_t D, int32_t bs, int32_t num_blocks, double scale,
                           double* out)
{
    return attention_rows(q, k_pool, NULL, NULL, v_pool, block_tables, max_blocks_per_seq,
                          context_lens, B, q_len, Hq, Hkv, D, bs, num_blocks, scale, out);
}

/*
 * Quantised K pool.  [T2] §"KV Cache量化": INT8 KV caches; keys are quantised
 * per channel (KVQuant), because their distribution is uneven across
 * channels.  [T3] §4.2: keys per channel at low bit width, values stay FP16.
 * Reading (the printed pseudo-code divides the maximum by 2^bits - 1 but
 * clamps to the signed range, and takes a signed maximum): symmetric 8-bit
 * codes, one scale per (KV head, channel) fixed from calibration tokens,
 *   scale[h][d] = max_t |K[t][h][d]| / 127   (1 for an all-zero channel),
 *   code = clamp(rint(k / scale), -128, 127),   K~ = code * scale.
 * Codes are integers decided by floating point, so they are computed in the
 * kernel's precision: fp32, correctly rounded division, round half to even.
 * The pages say nothing of non-finite keys: +-inf clamp like any large value,
 * and a NaN (e.g. an unwritten slot, never attended) stores code 0.
 * Code pool: int8 [num_blocks][Hkv][bs][D]; scales: fp32 [Hkv][D].
 */
int oracle_k_scales(const uint16_t* k, int64_t T, int32_t Hkv, int32_t D, float* scales)
{
    if (T < 0 || Hkv < 1 || D < 1) return ORACLE_ERR_ARG;
    for (int32_t h = 0; h < Hkv; ++h)
        for (int32_t d = 0; d < D; ++d) {
            double amax = 0.0;
            for (int64_t t = 0; t < T; ++t) {
                const double v = fabs(oracle_half_to_double(k[((size_t)t * Hkv + h) * D + d]));
                if (v > amax) amax = v;
            }
            /* |fp16| is exact in fp32; one correctly rounded fp32 division */
            scales[(size_t)h * D + d] = amax > 0.0 ? (float)amax / 127.0f : 1.0f;
        }
    return ORACLE_OK;
}

static int8_t k_code(uint16_t k, float scale)
{
    const float r = rintf((float)oracle_half_to_double(k) / scale);
    if (isnan(r)) return 0; /* a NaN key (an unwritten slot) stores code 0 */
    return (int8_t)(r < -128.0f ? -128.0f : (r > 127.0f ? 127.0f : r));
}

int oracle_append_q8k(const uint16_t* new_k, const uint16_t* new_v, const int64_t* slot_mapping,
                      int32_t T, int32_t Hkv, int32_t D, int32_t bs, int32_t num_blocks,
                      const float* k_scales, int8_t* kq_pool, uint16_t* v_pool)
{
    for (int32_t t = 0; t < T; ++t)
        if (slot_mapping[t] >= (int64_t)num_blocks * bs) return ORACLE_ERR_ARG;
    for (int32_t t = 0; t < T; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t p = slot / bs;
        int32_t o = (int32_t)(slot % bs);
        for (int32_t h = 0; h < Hkv; ++h) {
            for (int32_t d = 0; d < D; ++d) {
                const size_t src = ((size_t)t * Hkv + h) * D + d;
                kq_pool[pool_row(p, h, o, Hkv, bs, D) + d] = k_code(new_k[src], k_scales[(size_t)h * D + d]);
                v_pool[pool_row(p, h, o, Hkv, bs, D) + d] = new_v[src];
            }
        }
    }
    return ORACLE_OK;
}

int oracle_paged_attention_q8k(const uint16_t* q, const int8_t* kq_pool, const float* k_scales,
                               const uint16_t* v_pool, const int32_t* block_tables,
                               int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t B,
                               int32_t q_len, int32_t Hq, int32_t Hkv, int32_t D, int32_t bs,
                               int32_t num_blocks, double scale, double* out)
{
    return attention_rows(q, NULL, kq_pool, k_scales, v_pool, block_tables, max_blocks_per_seq,
                          context_lens, B, q_len, Hq, Hkv, D, bs, num_blocks, scale, out);
}

/*
 * Cache append: for every new token t with slot_mapping[t] >= 0,
 *   pool[slot / bs][h][slot % bs][:] = new[t][h][:]   for every KV head h,
 * for the K pool and the V pool alike.  Every other byte is left as it was.
 * new_k / new_v: [T][Hkv][D].  Returns ORACLE_ERR_ARG if a slot lies beyond the
 * pool (nothing is written in that case).
 */
int oracle_append(const uint16_t* new_k, const uint16_t* new_v, const int64_t* slot_mapping,
                  int32_t T, int32_t Hkv, int32_t D, int32_t bs, int32_t num_blocks,
                  uint16_t* k_pool, uint16_t* v_pool)
{
    for (int32_t t = 0; t < T; ++t)
        if (slot_mapping[t] >= (int64_t)num_blocks * bs) return ORACLE_ERR_ARG;
    for (int32_t t = 0; t < T; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t p = slot / bs;
        int32_t o = (int32_t)(slot % bs);
        for (int32_t h = 0; h < Hkv; ++h) {
            for (int32_t d = 0; d < D; ++d) {
                k_pool[pool_row(p, h, o, Hkv, bs, D) + d] = new_k[((size_t)t * Hkv + h) * D + d];
                v_pool[pool_row(p, h, o, Hkv, bs, D) + d] = new_v[((size_t)t * Hkv + h) * D + d];
            }
        }
    }
    return ORACLE_OK;
}

/*
 * Copy-on-write block copy: for each pair i, physical block pairs[2i+1] of
 * both pools becomes a byte copy of block pairs[2i] (every head, every slot).
 * Pairs are applied in order.
 */
int oracle_copy_blocks(const int32_t* pairs, int32_t n, int32_t Hkv, int32_t D, int32_t bs,
                       int32_t num_blocks, uint16_t* k_pool, uint16_t* v_pool)
{
    for (int32_t i = 0; i < 2 * n; ++i)
        if (pairs[i] < 0 || pairs[i] >= num_blocks) return ORACLE_ERR_ARG;
    const size_t per_block = (size_t)Hkv * bs * D;
    for (int32_t i = 0; i < n; ++i) {
        size_t src = (size_t)pairs[2 * i] * per_block;
        size_t dst = (size_t)pairs[2 * i + 1] * per_block;
        for (size_t e = 0; e < per_block; ++e) {
            k_pool[dst + e] = k_pool[src + e];
            v_pool[dst + e] = v_pool[src + e];
        }
    }
    return ORACLE_OK;
}
