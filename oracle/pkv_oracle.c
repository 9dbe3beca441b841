/*
 * pkv_oracle.c -- plain, slow, obviously correct fp64 CPU oracle for the paged KV-cache
 * decode path.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
 * baseline call it; the product library never links, loads or calls it, and it shares no
 * code, header, table or helper with the CUDA path.
 *
 * What it follows (page titles and sections of the source material):
 *   - "Memory Optimization in LLM Serving with PagedAttention", section "How PagedAttention
 *     Works": the KV cache is cut into fixed-size blocks (16 tokens by default), a sequence's
 *     logical blocks map to scattered physical blocks through a per-sequence block table, and
 *     the attention kernel gathers those scattered blocks to compute attention.
 *   - same page, section "Advanced Capabilities: Memory Sharing with Copy-on-Write": a write
 *     into a shared block first copies the block's whole content to a fresh block.
 *   - "vLLM and PagedAttention: How Ideas from Operating Systems Accelerated LLM Inference":
 *     16-token blocks by default, only the last block partly filled, custom kernels that work
 *     on scattered blocks.
 *
 * The attention these pages describe is never written out as a formula.  The plainest
 * reading, used here, is single-query softmax attention over every cached token of the
 * sequence:  x_t = scale * <q, K_t>,  out = sum_t exp(x_t - M) V_t / sum_t exp(x_t - M)
 * with M = max_t x_t, computed as an exact two-pass softmax in double precision, no split,
 * no running rescale, no blocking.
 *
 * Readings of points the pages leave open (each also listed in the design notes):
 *   - pool layout [num_blocks, num_kv_heads, block_size, head_dim], row-major;
 *   - token t of sequence s lives at physical block block_tables[s][t / block_size],
 *     offset t % block_size; only the first ceil(len / block_size) table entries are read;
 *   - query head h reads KV head h / (num_q_heads / num_kv_heads) (consecutive grouping);
 *   - 16-bit inputs are the exact values their bit patterns encode (IEEE binary16, bfloat16);
 *   - slot s of the pool means block s / block_size, offset s % block_size; slot -1 = skip.
 *
 * Parity pins for everything here live in the tests (brute-force contiguous attention,
 * closed forms, placement-permutation invariance, the split/merge identity, worked examples).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* dtype codes understood by this file (the Python wrapper maps names to them) */
#define ORC_F32 0
#define ORC_F16 1
#define ORC_BF16 2

#define ORC_OK 0
#define ORC_BAD_ARG 1
#define ORC_BAD_LEN 2
#define ORC_BAD_BLOCK 3
#define ORC_BAD_SLOT 4
#define ORC_NO_MEM 5

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double orc_f16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^(1-15-10) */
    } else if (e == 31) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + f), e - 25);     /* (1 + f/2^10) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double orc_bf16_to_f64(uint16_t b) {
    int sign = (b >> 15) & 1;
    int e = (b >> 7) & 0xff;
    int f = b & 0x7f;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -133);                /* subnormal: f * 2^(1-127-7) */
    } else if (e == 255) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(128 + f), e - 134);     /* (1 + f/2^7) * 2^(e-127) */
    }
    return sign ? -v : v;
}

static double orc_load(const void *base, int dtype, size_t i) {
    switch (dtype) {
    case ORC_F32: return (double)((const float *)base)[i];
    case ORC_F16: return orc_f16_to_f64(((const uint16_t *)base)[i]);
    case ORC_BF16: return orc_bf16_to_f64(((const uint16_t *)base)[i]);
    default: return NAN;
    }
}

static int orc_elem_size(int dtype) {
    return dtype == ORC_F32 ? 4 : (dtype == ORC_F16 || dtype == ORC_BF16) ? 2 : 0;
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Index of element (token offset o, dim d) of KV head hk in physical block p. */
static size_t orc_kv_index(int64_t p, int hk, int o, int d, int Hkv, int B, int D) {
    return (((size_t)p * Hkv + hk) * B + o) * D + d;
}

/*
 * Check that sequence s can be gathered: 1 <= len <= maxB*B and every table entry it needs
 * names a block in [0, NB).
 */
static int orc_check_seq(int s, int B, int NB, int maxB, const int32_t *bt, const int32_t *lens) {
    int L = lens[s];
    if (L < 1 || (int64_t)L > (int64_t)maxB * B) return ORC_BAD_LEN;
    int nblk = (L + B - 1) / B;
    for (int j = 0; j < nblk; ++j) {
        int32_t p = bt[(size_t)s * maxB + j];
        if (p < 0 || p >= NB) return ORC_BAD_BLOCK;
    }
    return ORC_OK;
}

/*
 * One (sequence, query head) row of decode attention, exact two-pass softmax in fp64.
 * out_row receives D doubles.
 */
static int orc_attn_row(int s, int h, int Hq, int Hkv, int D, int B, int NB, int maxB,
                        const void *q, int q_dtype, const void *k_pool, const void *v_pool,
                        int kv_dtype, const int32_t *bt, const int32_t *lens, double scale,
                        double *out_row) {
    int rc = orc_check_seq(s, B, NB, maxB, bt, lens);
    if (rc) return rc;
    int L = lens[s];
    int g = Hq / Hkv;
    int hk = h / g;

    double *qv = (double *)malloc(sizeof(double) * (size_t)D);
    double *x = (double *)malloc(sizeof(double) * (size_t)L);
    if (!qv || !x) { free(qv); free(x); return ORC_NO_MEM; }
    for (int d = 0; d < D; ++d) qv[d] = orc_load(q, q_dtype, ((size_t)s * Hq + h) * D + d);

    /* pass 1: scores through the block table, and their maximum */
    double M = -INFINITY;
    for (int t = 0; t < L; ++t) {
        int64_t p = bt[(size_t)s * maxB + t / B];
        int o = t % B;
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += qv[d] * orc_load(k_pool, kv_dtype, orc_kv_index(p, hk, o, d, Hkv, B, D));
        x[t] = scale * acc;
        if (x[t] > M) M = x[t];
    }
    /* pass 2: weights and the weighted sum of V */
    double den = 0.0;
    for (int d = 0; d < D; ++d) out_row[d] = 0.0;
    for (int t = 0; t < L; ++t) {
        int64_t p = bt[(size_t)s * maxB + t / B];
        int o = t % B;
        double w = exp(x[t] - M);
        den += w;
        for (int d = 0; d < D; ++d)
            out_row[d] += w * orc_load(v_pool, kv_dtype, orc_kv_index(p, hk, o, d, Hkv, B, D));
    }
    for (int d = 0; d < D; ++d) out_row[d] /= den;
    free(qv);
    free(x);
    return ORC_OK;
}

/*
 * Decode attention for a list of (sequence, query head) rows.
 *   rows: int32 pairs [nrows][2] = (s, h); NULL means every row in order s-major, h-minor
 *         (nrows is then ignored and S*Hq rows are written).
 *   out:  double [nrows][D].
 * Returns ORC_OK or the first error found (rows are independent; an error row is NaN).
 */
int orc_paged_attn_decode(int S, int Hq, int Hkv, int D, int B, int NB, int maxB,
                          const void *q, int q_dtype, const void *k_pool, const void *v_pool,
                          int kv_dtype, const int32_t *block_tables, const int32_t *context_lens,
                          double scale, const int32_t *rows, int nrows, double *out,
                          int nthreads) {
    if (S < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || D < 1 || B < 1 || NB < 0 || maxB < 0)
        return ORC_BAD_ARG;
    if (!orc_elem_size(q_dtype) || !orc_elem_size(kv_dtype)) return ORC_BAD_ARG;
    int n = rows ? nrows : S * Hq;
    int err = ORC_OK;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int r = 0; r < n; ++r) {
        int s = rows ? rows[2 * r] : r / Hq;
        int h = rows ? rows[2 * r + 1] : r % Hq;
        int rc;
        if (s < 0 || s >= S || h < 0 || h >= Hq) rc = ORC_BAD_ARG;
        else rc = orc_attn_row(s, h, Hq, Hkv, D, B, NB, maxB, q, q_dtype, k_pool, v_pool,
                               kv_dtype, block_tables, context_lens, scale,
                               out + (size_t)r * D);
        if (rc) {
            for (int d = 0; d < D; ++d) out[(size_t)r * D + d] = NAN;
#pragma omp critical
            { if (!err) err = rc; }
        }
    }
    return err;
}

/*
 * Split-context form of the same attention, written from its definition so that tests can
 * check that cutting the context into partitions and merging them by log-sum-exp gives the
 * one-pass result.  For partition p = tokens [p*P, min(L, (p+1)*P)):
 *   m_p = max x_t,  l_p = sum exp(x_t - m_p),  o_p = sum exp(x_t - m_p) V_t
 * and the merge is  out = sum_p exp(m_p - M) o_p / sum_p exp(m_p - M) l_p,  M = max_p m_p.
 * partials (optional, may be NULL): double [num_partitions][D + 2] = (o_p..., m_p, l_p) for
 * the single row (s, h).
 */
int orc_split_lse_row(int s, int h, int S, int Hq, int Hkv, int D, int B, int NB, int maxB,
                      const void *q, int q_dtype, const void *k_pool, const void *v_pool,
                      int kv_dtype, const int32_t *block_tables, const int32_t *context_lens,
                      double scale, int P, double *out_row, double *partials) {
    if (s < 0 || s >= S || h < 0 || h >= Hq || Hq % Hkv || P < 1) return ORC_BAD_ARG;
    int rc = orc_check_seq(s, B, NB, maxB, block_tables, context_lens);
    if (rc) return rc;
    int L = context_lens[s];
    int hk = h / (Hq / Hkv);
    int np = (L + P - 1) / P;
    double *m = (double *)malloc(sizeof(double) * np);
    double *l = (double *)malloc(sizeof(double) * np);
    double *o = (double *)calloc((size_t)np * D, sizeof(double));
    double *x = (double *)malloc(sizeof(double) * P);
    if (!m || !l || !o || !x) { free(m); free(l); free(o); free(x); return ORC_NO_MEM; }
    for (int p = 0; p < np; ++p) {
        int t0 = p * P, t1 = t0 + P < L ? t0 + P : L;
        m[p] = -INFINITY;
        for (int t = t0; t < t1; ++t) {
            int64_t blk = block_tables[(size_t)s * maxB + t / B];
            double acc = 0.0;
            for (int d = 0; d < D; ++d)
                acc += orc_load(q, q_dtype, ((size_t)s * Hq + h) * D + d) *
                       orc_load(k_pool, kv_dtype, orc_kv_index(blk, hk, t % B, d, Hkv, B, D));
            x[t - t0] = scale * acc;
            if (x[t - t0] > m[p]) m[p] = x[t - t0];
        }
        l[p] = 0.0;
        for (int t = t0; t < t1; ++t) {
            int64_t blk = block_tables[(size_t)s * maxB + t / B];
            double w = exp(x[t - t0] - m[p]);
            l[p] += w;
            for (int d = 0; d < D; ++d)
                o[(size_t)p * D + d] +=
                    w * orc_load(v_pool, kv_dtype, orc_kv_index(blk, hk, t % B, d, Hkv, B, D));
        }
        if (partials) {
            for (int d = 0; d < D; ++d) partials[(size_t)p * (D + 2) + d] = o[(size_t)p * D + d];
            partials[(size_t)p * (D + 2) + D] = m[p];
            partials[(size_t)p * (D + 2) + D + 1] = l[p];
        }
    }
    double Mx = -INFINITY;
    for (int p = 0; p < np; ++p) if (m[p] > Mx) Mx = m[p];
    double den = 0.0;
    for (int d = 0; d < D; ++d) out_row[d] = 0.0;
    for (int p = 0; p < np; ++p) {
        double c = exp(m[p] - Mx);
        den += c * l[p];
        for (int d = 0; d < D; ++d) out_row[d] += c * o[(size_t)p * D + d];
    }
    for (int d = 0; d < D; ++d) out_row[d] /= den;
    free(m); free(l); free(o); free(x);
    return ORC_OK;
}

/*
 * Write each new token's K and V into its slot: for token t and KV head h,
 *   pool[slot / B, h, slot % B, :] := new[t, h, :]   (bytes copied unchanged)
 * slot -1 means "skip this token".  Any other slot outside [0, NB*B) is an error and
 * nothing is written for that token.
 */
int orc_kv_write(int T, int Hkv, int D, int B, int NB, int elem_size, const void *k_new,
                 const void *v_new, const int64_t *slot_mapping, void *k_pool, void *v_pool) {
    if (T < 0 || Hkv < 1 || D < 1 || B < 1 || NB < 0 || elem_size < 1) return ORC_BAD_ARG;
    int err = ORC_OK;
    size_t row = (size_t)D * elem_size;
    for (int t = 0; t < T; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot == -1) continue;
        if (slot < 0 || slot >= (int64_t)NB * B) { err = ORC_BAD_SLOT; continue; }
        int64_t blk = slot / B;
        int off = (int)(slot % B);
        for (int h = 0; h < Hkv; ++h) {
            size_t dst = orc_kv_index(blk, h, off, 0, Hkv, B, D) * elem_size;
            size_t src = ((size_t)t * Hkv + h) * row;
            memcpy((char *)k_pool + dst, (const char *)k_new + src, row);
            memcpy((char *)v_pool + dst, (const char *)v_new + src, row);
        }
    }
    return err;
}

/*
 * Copy-on-write block copy: for each pair (src, dst), the whole physical block dst of both
 * pools (every KV head, every slot) becomes a byte copy of block src.  Pairs are applied in
 * order; a pair naming a block outside [0, NB) is an error and is skipped.
 */
int orc_kv_copy_blocks(int P, const int32_t *pairs, int Hkv, int D, int B, int NB,
                       int elem_size, void *k_pool, void *v_pool) {
    if (P < 0 || Hkv < 1 || D < 1 || B < 1 || NB < 0 || elem_size < 1) return ORC_BAD_ARG;
    int err = ORC_OK;
    size_t blk_bytes = (size_t)Hkv * B * D * elem_size;
    for (int i = 0; i < P; ++i) {
        int32_t src = pairs[2 * i], dst = pairs[2 * i + 1];
        if (src < 0 || src >= NB || dst < 0 || dst >= NB) { err = ORC_BAD_BLOCK; continue; }
        memmove((char *)k_pool + (size_t)dst * blk_bytes,
                (const char *)k_pool + (size_t)src * blk_bytes, blk_bytes);
        memmove((char *)v_pool + (size_t)dst * blk_bytes,
                (const char *)v_pool + (size_t)src * blk_bytes, blk_bytes);
    }
    return err;
}

/*
 * Swap copy between two pools of equal block shape (a device pool and a host pool): for each
 * pair (src, dst), block dst of the destination pools becomes a byte copy of block src of the
 * source pools, for K and V.  "vLLM and PagedAttention: How Ideas from Operating Systems
 * Accelerated LLM Inference": evicted sequences are swapped to CPU memory and back.
 */
int orc_kv_swap(int P, const int32_t *pairs, const void *src_k, const void *src_v, int nb_src,
                void *dst_k, void *dst_v, int nb_dst, size_t block_bytes) {
    if (P < 0 || nb_src < 0 || nb_dst < 0) return ORC_BAD_ARG;
    int err = ORC_OK;
    for (int i = 0; i < P; ++i) {
        int32_t s = pairs[2 * i], d = pairs[2 * i + 1];
        if (s < 0 || s >= nb_src || d < 0 || d >= nb_dst) { err = ORC_BAD_BLOCK; continue; }
        memcpy((char *)dst_k + (size_t)d * block_bytes, (const char *)src_k + (size_t)s * block_bytes,
               block_bytes);
        memcpy((char *)dst_v + (size_t)d * block_bytes, (const char *)src_v + (size_t)s * block_bytes,
               block_bytes);
    }
    return err;
}

/* ---------------------------------------------------------------------------------------
 * FP8 (E4M3) KV cache.  "Memory Optimization in LLM Serving with PagedAttention", section
 * "Broader Context: vLLM, TGI, and TensorRT-LLM": paged KV caches are also kept in INT8/FP8
 * to cut memory.  The scheme (our reading; the page names no format): each KV head has one
 * fp32 scale for K and one for V; a value x is stored as the E4M3 code of x / scale (fp32
 * division, round to nearest even, saturating to +-448); its value is code * scale.
 * K blocks keep the [block][head][token][dim] layout; V blocks are stored transposed within
 * the block, [block][head][dim][slot], slot p holding token 2*(p/4) + p%2 + 8*((p/2)%2).
 * ------------------------------------------------------------------------------------- */

/* E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 fraction bits; no infinities; S.1111.111 is
 * NaN; largest finite 448. */
double orc_e4m3_to_f64(uint8_t c) {
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 0xf;
    int f = c & 0x7;
    double v;
    if (e == 15 && f == 7) return NAN;
    if (e == 0) v = ldexp((double)f, -9);              /* f * 2^(1-7-3) */
    else v = ldexp((double)(8 + f), e - 10);           /* (1 + f/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* Nearest E4M3 code of a float (ties to even), saturating to +-448; NaN gives 0x7F. */
uint8_t orc_f32_to_e4m3(float x) {
    if (x != x) return 0x7f;
    uint8_t sign = (x < 0 || (x == 0 && signbit(x))) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7e;
    int code;
    if (a < ldexp(1.0, -6)) {
        /* subnormal grid, step 2^-9; the carry out of 7 is the smallest normal code 8 */
        code = (int)nearbyint(a / ldexp(1.0, -9));
    } else {
        int ex;
        frexp(a, &ex);                                /* a = m * 2^ex, m in [0.5, 1) */
        int e = ex - 1;                               /* a in [2^e, 2^(e+1)) */
        int n = (int)nearbyint(a / ldexp(1.0, e - 3)); /* in [8, 16] */
        code = ((e + 7) << 3) + (n - 8);              /* n = 16 carries into e + 1 */
    }
    if (code > 0x7e) code = 0x7e;
    return sign | (uint8_t)code;
}

/* Transposed V rows hold the block's 16 tokens in a fixed slot order: slot p holds token
 * 2*(p/4) + p%2 + 8*((p/2)%2).  The slot of token t is found by trying every slot. */
static int orc_v_slot(int t) {
    for (int p = 0; p < 16; ++p)
        if (2 * (p / 4) + p % 2 + 8 * ((p / 2) % 2) == t) return p;
    return -1;
}

/* Value of new element i of dtype (f16 / bf16 / f32) as a float (exact). */
static float orc_load_f32(const void *base, int dtype, size_t i) {
    return (float)orc_load(base, dtype, i);
}

/*
 * Byte offset of token `off` (of a B-token block), dim d, in the FP8 V pool
 * [NB][Hkv][B/16][D][16]: every 16-token half of a block is stored transposed, its row of
 * 16 slots in the slot order above.  With B = 16 this is [NB][Hkv][D][16].
 */
static size_t orc_v_fp8_index(int64_t blk, int h, int off, int d, int Hkv, int B, int D) {
    return ((((size_t)blk * Hkv + h) * (size_t)(B / 16) + (size_t)(off / 16)) * D + d) * 16 +
           (size_t)orc_v_slot(off % 16);
}

/*
 * kv_write into FP8 pools (B a multiple of 16): for token t and head h with slot s
 * (s = -1 skips),
 *   k_pool[s/B][h][s%B][d] = e4m3(k_new[t][h][d] / k_scale[h])
 *   v_pool at orc_v_fp8_index(s/B, h, s%B, d) = e4m3(v_new[t][h][d] / v_scale[h])
 */
int orc_kv_write_fp8(int T, int Hkv, int D, int B, int NB, const void *k_new,
                     const void *v_new, int new_dtype, const int64_t *slot_mapping,
                     const float *k_scale, const float *v_scale, uint8_t *k_pool,
                     uint8_t *v_pool) {
    if (T < 0 || Hkv < 1 || D < 1 || B < 16 || B % 16 || NB < 0 || !orc_elem_size(new_dtype))
        return ORC_BAD_ARG;
    int err = ORC_OK;
    for (int t = 0; t < T; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot == -1) continue;
        if (slot < 0 || slot >= (int64_t)NB * B) { err = ORC_BAD_SLOT; continue; }
        int64_t blk = slot / B;
        int off = (int)(slot % B);
        for (int h = 0; h < Hkv; ++h)
            for (int d = 0; d < D; ++d) {
                size_t src = ((size_t)t * Hkv + h) * D + d;
                float kq = orc_load_f32(k_new, new_dtype, src) / k_scale[h];
                float vq = orc_load_f32(v_new, new_dtype, src) / v_scale[h];
                k_pool[(((size_t)blk * Hkv + h) * B + off) * D + d] = orc_f32_to_e4m3(kq);
                v_pool[orc_v_fp8_index(blk, h, off, d, Hkv, B, D)] = orc_f32_to_e4m3(vq);
            }
    }
    return err;
}

/* Decode attention over FP8 pools (layouts above), exact two-pass softmax in fp64 on the
 * dequantised values code * scale.  Same row contract as orc_paged_attn_decode. */
int orc_paged_attn_decode_fp8(int S, int Hq, int Hkv, int D, int B, int NB, int maxB,
                              const void *q, int q_dtype, const uint8_t *k_pool,
                              const uint8_t *v_pool, const float *k_scale,
                              const float *v_scale, const int32_t *block_tables,
                              const int32_t *context_lens, double scale, const int32_t *rows,
                              int nrows, double *out, int nthreads) {
    if (S < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || D < 1 || B < 16 || B % 16 || NB < 0 ||
        maxB < 0 || !orc_elem_size(q_dtype))
        return ORC_BAD_ARG;
    int n = rows ? nrows : S * Hq;
    int err = ORC_OK;
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int r = 0; r < n; ++r) {
        int s = rows ? rows[2 * r] : r / Hq;
        int h = rows ? rows[2 * r + 1] : r % Hq;
        double *o = out + (size_t)r * D;
        int rc = (s < 0 || s >= S || h < 0 || h >= Hq) ? ORC_BAD_ARG
                 : orc_check_seq(s, B, NB, maxB, block_tables, context_lens);
        if (rc) {
            for (int d = 0; d < D; ++d) o[d] = NAN;
#pragma omp critical
            { if (!err) err = rc; }
            continue;
        }
        int L = context_lens[s], hk = h / (Hq / Hkv);
        double ks = k_scale[hk], vs = v_scale[hk];
        double *x = (double *)malloc(sizeof(double) * (size_t)L);
        double M = -INFINITY;
        for (int t = 0; t < L; ++t) {
            int64_t p = block_tables[(size_t)s * maxB + t / B];
            double acc = 0.0;
            for (int d = 0; d < D; ++d)
                acc += orc_load(q, q_dtype, ((size_t)s * Hq + h) * D + d) *
                       (orc_e4m3_to_f64(k_pool[(((size_t)p * Hkv + hk) * B + t % B) * D + d]) * ks);
            x[t] = scale * acc;
            if (x[t] > M) M = x[t];
        }
        double den = 0.0;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        for (int t = 0; t < L; ++t) {
            int64_t p = block_tables[(size_t)s * maxB + t / B];
            double w = exp(x[t] - M);
            den += w;
            for (int d = 0; d < D; ++d)
                o[d] += w * (orc_e4m3_to_f64(
                                 v_pool[orc_v_fp8_index(p, hk, t % B, d, Hkv, B, D)]) * vs);
        }
        for (int d = 0; d < D; ++d) o[d] /= den;
        free(x);
    }
    return err;
}
