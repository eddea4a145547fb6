/*
 * gqa_oracle.c -- plain, slow, fp64 CPU oracle for grouped-query attention over a
 * paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or calls
 * this file; it is used by tests/, by __graft_entry__.smoke() and by bench.py's CPU
 * baseline leg.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (sources, by page title and section):
 *   - GQA: Hq query heads split into Hk groups of g = Hq/Hk consecutive heads; each
 *     group reads one K/V head ("TensorRT对Grouped Query Attention的支持进展",
 *     section "技术演进背景：从MHA到GQA的必然选择").  Query head h reads KV head
 *     floor(h/g), the head a repeat_kv (repeat-interleave) copy would hand it
 *     (same page, section "图优化与算子融合", RepeatKVPlugin).
 *   - Paged KV cache: a sequence's logically contiguous KV lives in fixed-size pages
 *     scattered in a pool and is found through a per-sequence page table
 *     ("TensorRT-LLM与TensorRT核心差异解析", section 4.2.2 PageAttention; and
 *     "TensorRT对Grouped Query Attention的支持进展", section "动态形状与KV Cache管理":
 *     the caller keeps the pool and passes the physical page indices).
 *   - The attention itself is plain softmax(q K^T * scale) V: fused/tiled kernels reach
 *     the same result as the decomposed MatMul -> Softmax -> MatMul form
 *     ("TensorRT-LLM与TensorRT核心差异解析", sections 4.1 and 4.2.1 FlashAttention).
 *     The oracle IS the decomposed form, in fp64, with no tiling and no online softmax.
 *   - NumSplits: the attention over the KV length is split into sub-problems and merged
 *     ("解锁GQA性能潜力：从批量大小敏感性到高效优化实践", section "核心参数调优：PackGQA与
 *     NumSplits的协同舞蹈").  The oracle merges splits by their log-sum-exp.
 *   - Causal chunked prefill: a chunk of new query tokens appended after a paged prior
 *     context ("TensorRT对Grouped Query Attention的支持进展", section
 *     "与动态批处理协同", chunked prefill).  Row i of a chunk of Lq tokens in a sequence
 *     of total length L sits at absolute position L - Lq + i and sees keys 0..pos.
 *   - FP8 KV: e4m3 codes times a per-(page, kv head) scale ("解锁GQA性能潜力…",
 *     section "实践验证：从理论到落地的性能跃迁", FP8).  Decoded here from the OCP
 *     FP8 E4M3 format definition.
 *
 * Layouts (all row-major, C order):
 *   q        : uint16 bf16 bits [B][Hq][D]           (decode)   or [total_q][Hq][D] (prefill)
 *   k_pages  : [num_pages][Hk][P][D]  elements of kv_dtype (0 = bf16 bits, 1 = e4m3 bytes)
 *   v_pages  : same as k_pages
 *   k_scale  : double [num_pages][Hk] (fp8 only; NULL for bf16)
 *   page_table: int32 [B][pt_stride]; entry p of row b is the physical page of logical page p
 *   seq_lens : int32 [B]; length of sequence b including the current token(s)
 *   out      : double [rows][Hq][D];  lse : double [rows][Hq] (natural log)
 *
 * An empty sequence (L = 0) has output 0 and lse = -inf.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 is the upper half of an IEEE-754 binary32: 1 sign bit, 8 exponent bits
 * (bias 127), 7 fraction bits. */
double oracle_bf16_to_f64(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int e = (bits >> 7) & 0xff;
    int f = bits & 0x7f;
    double v;
    if (e == 0xff)
        v = f ? NAN : INFINITY;
    else if (e == 0)
        v = ldexp((double)f, -126 - 7); /* subnormal: 0.f * 2^-126 */
    else
        v = ldexp(1.0 + (double)f / 128.0, e - 127);
    return sign ? -v : v;
}

/* OCP FP8 E4M3 ("fn" variant): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits,
 * no infinities, S.1111.111 is NaN, largest finite 448. */
double oracle_e4m3_to_f64(uint8_t bits)
{
    int sign = (bits >> 7) & 1;
    int e = (bits >> 3) & 0xf;
    int m = bits & 0x7;
    double v;
    if (e == 0xf && m == 7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m, -6 - 3); /* subnormal: 0.m * 2^-6 */
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Value of element (phys, kvh, slot, d) of a page pool, dequantised. */
static double kv_value(const void *pages, int kv_dtype, const double *scale, int Hk, int P,
                       int D, int64_t phys, int kvh, int slot, int d)
{
    int64_t idx = (((phys * Hk) + kvh) * (int64_t)P + slot) * D + d;
    if (kv_dtype == 0)
        return oracle_bf16_to_f64(((const uint16_t *)pages)[idx]);
    return oracle_e4m3_to_f64(((const uint8_t *)pages)[idx]) * scale[phys * Hk + kvh];
}

/* Step 1 of the definition: copy sequence b's keys (or values) for KV head kvh out of
 * the pool into a contiguous [L][D] fp64 array, token t living in logical page t / P at
 * slot t % P. */
static void gather_f64(const void *pages, int kv_dtype, const double *scale,
                       const int32_t *page_table, int pt_stride, int b, int kvh, int L,
                       int Hk, int P, int D, double *dst)
{
    for (int t = 0; t < L; ++t) {
        int64_t phys = page_table[(int64_t)b * pt_stride + t / P];
        for (int d = 0; d < D; ++d)
            dst[(int64_t)t * D + d] = kv_value(pages, kv_dtype, scale, Hk, P, D, phys, kvh, t % P, d);
    }
}

/* Softmax attention of one query row against keys/values [t0, t1) of a contiguous copy:
 *   s_t = scale * <q, K_t>,  m = max s_t,  Z = sum exp(s_t - m),
 *   o = sum exp(s_t - m) V_t / Z,  lse = m + ln Z.
 * An empty range gives o = 0, lse = -inf. */
static void attend_row(const double *q, const double *K, const double *V, int t0, int t1, int D,
                       double scale, double *s, double *o, double *lse)
{
    for (int d = 0; d < D; ++d)
        o[d] = 0.0;
    if (t1 <= t0) {
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int t = t0; t < t1; ++t) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += q[d] * K[(int64_t)t * D + d];
        s[t] = scale * acc;
        if (s[t] > m)
            m = s[t];
    }
    double Z = 0.0;
    for (int t = t0; t < t1; ++t)
        Z += exp(s[t] - m);
    for (int t = t0; t < t1; ++t) {
        double w = exp(s[t] - m) / Z;
        for (int d = 0; d < D; ++d)
            o[d] += w * V[(int64_t)t * D + d];
    }
    *lse = m + log(Z);
}

static double *scales_f64(const float *s, int64_t n)
{
    if (!s)
        return NULL;
    double *r = (double *)malloc(sizeof(double) * (size_t)n);
    for (int64_t i = 0; i < n; ++i)
        r[i] = (double)s[i];
    return r;
}

/* Bit-exact contiguous copy-out of the cache: k_out/v_out[(cu_kv[b] + t)][kvh][d] equals
 * the pool element of token t of sequence b.  elem_bytes is 1 or 2; bytes are copied,
 * never interpreted. */
void oracle_gather(const void *k_pages, const void *v_pages, const int32_t *page_table,
                   int pt_stride, const int32_t *seq_lens, const int64_t *cu_kv, int B, int Hk,
                   int D, int P, int elem_bytes, void *k_out, void *v_out)
{
    size_t row = (size_t)D * (size_t)elem_bytes;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < seq_lens[b]; ++t) {
            int64_t phys = page_table[(int64_t)b * pt_stride + t / P];
            for (int kvh = 0; kvh < Hk; ++kvh) {
                size_t src = (size_t)(((phys * Hk) + kvh) * (int64_t)P + t % P) * row;
                size_t dst = (size_t)((cu_kv[b] + t) * Hk + kvh) * row;
                memcpy((char *)k_out + dst, (const char *)k_pages + src, row);
                memcpy((char *)v_out + dst, (const char *)v_pages + src, row);
            }
        }
}

/* Decode: one query token per sequence.  When num_splits > 0, the tokens of each
 * sequence are cut into num_splits contiguous, page-aligned ranges of ceil(np/num_splits)
 * pages (np = ceil(L/P)); split s covers tokens [s*c*P, min(L, (s+1)*c*P)).  Each split
 * gives its own normalised output and lse, written to o_part [S][B][Hq][D] and
 * lse_part [S][B][Hq].  When num_splits == 0 the whole sequence is one range and the
 * result goes to out [B][Hq][D], lse [B][Hq]. */
static void decode_impl(const uint16_t *q, const void *k_pages, const void *v_pages,
                        const float *k_scale_f, const float *v_scale_f, int kv_dtype,
                        const int32_t *page_table, int pt_stride, const int32_t *seq_lens,
                        int B, int Hq, int Hk, int D, int P, int num_pages, double scale,
                        int num_splits, double *out, double *lse)
{
    int g = Hq / Hk;
    int64_t nscale = (int64_t)num_pages * Hk;
    double *ks = scales_f64(k_scale_f, nscale), *vs = scales_f64(v_scale_f, nscale);
    int max_L = 0;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] > max_L)
            max_L = seq_lens[b];
#pragma omp parallel
    {
        double *K = (double *)malloc(sizeof(double) * ((size_t)max_L * D + 1));
        double *V = (double *)malloc(sizeof(double) * ((size_t)max_L * D + 1));
        double *s = (double *)malloc(sizeof(double) * ((size_t)max_L + 1));
        double *qd = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for collapse(2) schedule(dynamic)
        for (int b = 0; b < B; ++b)
            for (int kvh = 0; kvh < Hk; ++kvh) {
                int L = seq_lens[b];
                gather_f64(k_pages, kv_dtype, ks, page_table, pt_stride, b, kvh, L, Hk, P, D, K);
                gather_f64(v_pages, kv_dtype, vs, page_table, pt_stride, b, kvh, L, Hk, P, D, V);
                for (int j = 0; j < g; ++j) {
                    int h = kvh * g + j;
                    for (int d = 0; d < D; ++d)
                        qd[d] = oracle_bf16_to_f64(q[((int64_t)b * Hq + h) * D + d]);
                    if (num_splits == 0) {
                        attend_row(qd, K, V, 0, L, D, scale, s, out + ((int64_t)b * Hq + h) * D,
                                   lse + (int64_t)b * Hq + h);
                    } else {
                        int np = (L + P - 1) / P;
                        int c = (np + num_splits - 1) / num_splits;
                        for (int sp = 0; sp < num_splits; ++sp) {
                            int t0 = sp * c * P, t1 = (sp + 1) * c * P;
                            if (t1 > L)
                                t1 = L;
                            int64_t row = ((int64_t)sp * B + b) * Hq + h;
                            attend_row(qd, K, V, t0, t1, D, scale, s, out + row * D, lse + row);
                        }
                    }
                }
            }
        free(K);
        free(V);
        free(s);
        free(qd);
    }
    free(ks);
    free(vs);
}

void oracle_decode(const uint16_t *q, const void *k_pages, const void *v_pages,
                   const float *k_scale, const float *v_scale, int kv_dtype,
                   const int32_t *page_table, int pt_stride, const int32_t *seq_lens, int B,
                   int Hq, int Hk, int D, int P, int num_pages, double scale, double *out,
                   double *lse)
{
    decode_impl(q, k_pages, v_pages, k_scale, v_scale, kv_dtype, page_table, pt_stride,
                seq_lens, B, Hq, Hk, D, P, num_pages, scale, 0, out, lse);
}

void oracle_decode_split(const uint16_t *q, const void *k_pages, const void *v_pages,
                         const float *k_scale, const float *v_scale, int kv_dtype,
                         const int32_t *page_table, int pt_stride, const int32_t *seq_lens,
                         int B, int Hq, int Hk, int D, int P, int num_pages, double scale,
                         int num_splits, double *o_part, double *lse_part)
{
    decode_impl(q, k_pages, v_pages, k_scale, v_scale, kv_dtype, page_table, pt_stride,
                seq_lens, B, Hq, Hk, D, P, num_pages, scale, num_splits, o_part, lse_part);
}

/* Merge of split results by log-sum-exp: M = max_s lse_s, w_s = exp(lse_s - M),
 * O = sum w_s o_s / sum w_s, lse = M + ln sum w_s, the sums running over the non-empty
 * splits only: an empty split (lse = -inf) has no tokens, hence no output to weigh (its
 * o_s is undefined), and is left out.  All splits empty: O = 0, lse = -inf.
 * o_part [S][rows][D], lse_part [S][rows]. */
void oracle_lse_combine(const double *o_part, const double *lse_part, int S, int rows, int D,
                        double *out, double *lse)
{
    for (int r = 0; r < rows; ++r) {
        double M = -INFINITY;
        for (int s = 0; s < S; ++s)
            if (lse_part[(int64_t)s * rows + r] > M)
                M = lse_part[(int64_t)s * rows + r];
        for (int d = 0; d < D; ++d)
            out[(int64_t)r * D + d] = 0.0;
        if (M == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double W = 0.0;
        for (int s = 0; s < S; ++s) {
            if (lse_part[(int64_t)s * rows + r] == -INFINITY)
                continue;
            double w = exp(lse_part[(int64_t)s * rows + r] - M);
            W += w;
            for (int d = 0; d < D; ++d)
                out[(int64_t)r * D + d] += w * o_part[((int64_t)s * rows + r) * D + d];
        }
        for (int d = 0; d < D; ++d)
            out[(int64_t)r * D + d] /= W;
        lse[r] = M + log(W);
    }
}

/* Causal chunked prefill.  Sequence b owns query rows cu_q[b] .. cu_q[b+1]-1 (Lq rows)
 * and has L = seq_lens[b] >= Lq tokens in the cache, the chunk being the last Lq of
 * them.  Row i attends to keys 0 .. L-Lq+i when causal, to all L keys otherwise.
 * out [total_q][Hq][D], lse [total_q][Hq]. */
void oracle_prefill(const uint16_t *q, const int32_t *cu_q, const void *k_pages,
                    const void *v_pages, const float *k_scale_f, const float *v_scale_f,
                    int kv_dtype, const int32_t *page_table, int pt_stride,
                    const int32_t *seq_lens, int B, int Hq, int Hk, int D, int P, int num_pages,
                    double scale, int causal, double *out, double *lse)
{
    int g = Hq / Hk;
    int64_t nscale = (int64_t)num_pages * Hk;
    double *ks = scales_f64(k_scale_f, nscale), *vs = scales_f64(v_scale_f, nscale);
    int max_L = 0;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] > max_L)
            max_L = seq_lens[b];
#pragma omp parallel
    {
        double *K = (double *)malloc(sizeof(double) * ((size_t)max_L * D + 1));
        double *V = (double *)malloc(sizeof(double) * ((size_t)max_L * D + 1));
        double *s = (double *)malloc(sizeof(double) * ((size_t)max_L + 1));
        double *qd = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for collapse(2) schedule(dynamic)
        for (int b = 0; b < B; ++b)
            for (int kvh = 0; kvh < Hk; ++kvh) {
                int L = seq_lens[b];
                int Lq = cu_q[b + 1] - cu_q[b];
                gather_f64(k_pages, kv_dtype, ks, page_table, pt_stride, b, kvh, L, Hk, P, D, K);
                gather_f64(v_pages, kv_dtype, vs, page_table, pt_stride, b, kvh, L, Hk, P, D, V);
                for (int i = 0; i < Lq; ++i) {
                    int64_t qrow = cu_q[b] + i;
                    int t1 = causal ? (L - Lq + i + 1) : L;
                    for (int j = 0; j < g; ++j) {
                        int h = kvh * g + j;
                        for (int d = 0; d < D; ++d)
                            qd[d] = oracle_bf16_to_f64(q[(qrow * Hq + h) * D + d]);
                        attend_row(qd, K, V, 0, t1, D, scale, s, out + (qrow * Hq + h) * D,
                                   lse + qrow * Hq + h);
                    }
                }
            }
        free(K);
        free(V);
        free(s);
        free(qd);
    }
    free(ks);
    free(vs);
}

/* Number of threads an OpenMP parallel region of this library runs with. */
int oracle_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}

/* ---------------------------------------------------------------------------------------
 * KV append (the step before decode: "FasterTransformer source tour", where the fused
 * decoder step counts writing the new token into the KV cache among its three global
 * accesses; page layout as above).  Readings taken where the pages are silent:
 *   - seq_lens[b] already counts the new token, so it goes to position L_b - 1: page
 *     page_table[b][(L_b - 1) / P], slot (L_b - 1) % P, for every kv head.  L_b = 0
 *     appends nothing.
 *   - bf16 pools take the token's bits as given.
 *   - e4m3 pools: a token that opens a page (slot 0) sets that (page, kv head)'s scale
 *     to absmax / 448 in fp32 (1 for an all-zero token); a later token keeps the page's
 *     scale.  Each element becomes e4m3(x / scale), the quotient in fp32, rounded to
 *     nearest (ties to even) and saturated at +-448.
 * ------------------------------------------------------------------------------------- */

/* OCP e4m3 code of x: the nearest of the 127 non-negative finite codes by exhaustive
 * search (ties to the even code, i.e. mantissa LSB 0), with x's sign; magnitudes past 448
 * and infinities give +-448; NaN gives the NaN code 0x7f. */
uint8_t oracle_f32_to_e4m3(float x)
{
    if (isnan(x))
        return 0x7f;
    int sign = signbit(x) ? 1 : 0;
    if (isinf(x))
        return (uint8_t)((sign << 7) | 0x7e);
    double ax = fabs((double)x);
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c <= 0x7e; ++c) {
        double d = fabs(oracle_e4m3_to_f64((uint8_t)c) - ax);
        if (d < bd || (d == bd && (c & 1) == 0)) {
            bd = d;
            best = c;
        }
    }
    return (uint8_t)((sign << 7) | best);
}

static float bf16_bits_to_f32(uint16_t bits)
{
    return (float)oracle_bf16_to_f64(bits); /* exact: bf16 is a truncated binary32 */
}

void oracle_append_kv(void *k_pages, void *v_pages, float *k_scale, float *v_scale,
                      int kv_dtype, const int32_t *page_table, int pt_stride,
                      const int32_t *seq_lens, int B, int Hk, int D, int P,
                      const uint16_t *k_new, const uint16_t *v_new)
{
    for (int b = 0; b < B; ++b) {
        int L = seq_lens[b];
        if (L <= 0)
            continue;
        int t = L - 1;
        int64_t phys = page_table[(int64_t)b * pt_stride + t / P];
        int slot = t % P;
        for (int kvh = 0; kvh < Hk; ++kvh) {
            for (int which = 0; which < 2; ++which) {
                const uint16_t *src = (which == 0 ? k_new : v_new) + ((int64_t)b * Hk + kvh) * D;
                void *pages = which == 0 ? k_pages : v_pages;
                int64_t base = (((phys * Hk) + kvh) * (int64_t)P + slot) * D;
                if (kv_dtype == 0) {
                    for (int d = 0; d < D; ++d)
                        ((uint16_t *)pages)[base + d] = src[d];
                    continue;
                }
                float *scale = which == 0 ? k_scale : v_scale;
                int64_t si = phys * Hk + kvh;
                if (slot == 0) {
                    float amax = 0.0f;
                    for (int d = 0; d < D; ++d) {
                        float a = fabsf(bf16_bits_to_f32(src[d]));
                        if (a > amax)
                            amax = a;
                    }
                    scale[si] = amax > 0.0f ? amax / 448.0f : 1.0f;
                }
                float s = scale[si];
                for (int d = 0; d < D; ++d) {
                    float qv = bf16_bits_to_f32(src[d]) / s;
                    ((uint8_t *)pages)[base + d] = oracle_f32_to_e4m3(qv);
                }
            }
        }
    }
}

/* ---------------------------------------------------------------------------------------
 * Page-level top-K sparse decode: the decode stage of RocketKV as the page
 * "TensorRT-LLM 如何用 sparse_attention_config 配置 Sparse Attention 降低长上下文推理开销"
 * (RocketKV configuration section) describes it: an auxiliary KT cache scores the pages,
 * and the decode attends to the `topk` best pages plus the most recent `window` tokens
 * only.  Readings taken where the page is silent:
 *   - KT entry of (page, kv head): the element-wise minimum and maximum of the page's key
 *     vectors over its valid tokens.  kt[page][kvh][d][0] = min, [1] = max.
 *   - Score of a page for query head h: sum over d of max(q_d * min_d, q_d * max_d), the
 *     largest q.k over the box [min, max] and so an upper bound of q.k for every key of
 *     the page.  Score for a kv head: the sum of its g query heads' scores.  Computed in
 *     fp32, the decision's precision on the GPU: per head with d ascending, then heads
 *     ascending.  Every product of two bf16 values is exact in fp32, so both sides round
 *     the same sums the same way.
 *   - The selection unit is one KV-cache page (the page's sparse page_size taken equal to
 *     the cache's page size; the page asks for a power of two, which 16/32/64 are), and the
 *     query channels used are all head_dim of them (the page advises topr = head_dim).
 *   - Window: the pages holding any of the last `window` tokens are always attended.
 *     Among the earlier pages the `topk` highest scores are chosen, equal scores going to
 *     the lower logical page; with no more than `topk` earlier pages, all are chosen.
 *   - The attention itself is plain softmax attention over the tokens of the chosen
 *     pages (attend_row above), in logical page order.
 * ------------------------------------------------------------------------------------- */

/* KT entries of every page sequence b references: for page p < ceil(L/P), over its
 * n = min(P, L - p*P) valid tokens.  kt: double [num_pages][Hk][D][2] (caller-owned;
 * entries of unreferenced pages are left as they are). */
void oracle_kt_build(const uint16_t *k_pages, const int32_t *page_table, int pt_stride,
                     const int32_t *seq_lens, int B, int Hk, int D, int P, double *kt)
{
    for (int b = 0; b < B; ++b) {
        int L = seq_lens[b];
        int np = (L + P - 1) / P;
        for (int p = 0; p < np; ++p) {
            int64_t phys = page_table[(int64_t)b * pt_stride + p];
            int n = L - p * P < P ? L - p * P : P;
            for (int kvh = 0; kvh < Hk; ++kvh)
                for (int d = 0; d < D; ++d) {
                    double mn = INFINITY, mx = -INFINITY;
                    for (int t = 0; t < n; ++t) {
                        double v = kv_value(k_pages, 0, NULL, Hk, P, D, phys, kvh, t, d);
                        if (v < mn)
                            mn = v;
                        if (v > mx)
                            mx = v;
                    }
                    double *e = kt + ((phys * Hk + kvh) * (int64_t)D + d) * 2;
                    e[0] = mn;
                    e[1] = mx;
                }
        }
    }
}

/* Page scores: scores[b][kvh][p] for p < ceil(L_b/P) (fp32, as defined above); entries
 * at or past ceil(L_b/P) are set to -inf.  kt as built by oracle_kt_build. */
void oracle_page_scores(const uint16_t *q, const double *kt, const int32_t *page_table,
                        int pt_stride, const int32_t *seq_lens, int B, int Hq, int Hk, int D,
                        int P, float *scores)
{
    int g = Hq / Hk;
    for (int b = 0; b < B; ++b) {
        int L = seq_lens[b];
        int np = (L + P - 1) / P;
        for (int kvh = 0; kvh < Hk; ++kvh)
            for (int p = 0; p < pt_stride; ++p) {
                float *dst = scores + ((int64_t)b * Hk + kvh) * pt_stride + p;
                if (p >= np) {
                    *dst = -INFINITY;
                    continue;
                }
                int64_t phys = page_table[(int64_t)b * pt_stride + p];
                const double *e = kt + (phys * Hk + kvh) * (int64_t)D * 2;
                float total = 0.0f;
                for (int j = 0; j < g; ++j) {
                    int h = kvh * g + j;
                    float sh = 0.0f;
                    for (int d = 0; d < D; ++d) {
                        float qd = bf16_bits_to_f32(q[((int64_t)b * Hq + h) * D + d]);
                        float lo = qd * (float)e[2 * d], hi = qd * (float)e[2 * d + 1];
                        sh = sh + (lo > hi ? lo : hi);
                    }
                    total = total + sh;
                }
                *dst = total;
            }
    }
}

/* Selection from the scores: sel[b][kvh][0 .. nsel-1] = the chosen logical pages in
 * ascending order (window pages included), nsel[b][kvh] their count.  sel has pt_stride
 * entries per (b, kvh). */
void oracle_sparse_select(const float *scores, const int32_t *seq_lens, int B, int Hk,
                          int pt_stride, int P, int topk, int window, int32_t *sel,
                          int32_t *nsel)
{
    char *take = (char *)malloc((size_t)pt_stride + 1);
    for (int b = 0; b < B; ++b) {
        int L = seq_lens[b];
        int np = (L + P - 1) / P;
        int lo = L - window > 0 ? L - window : 0;
        int wp = window > 0 ? lo / P : np; /* first page holding a window token */
        if (wp > np)
            wp = np;
        for (int kvh = 0; kvh < Hk; ++kvh) {
            const float *s = scores + ((int64_t)b * Hk + kvh) * pt_stride;
            for (int p = 0; p < np; ++p)
                take[p] = p >= wp || wp <= topk;
            if (wp > topk) {
                /* topk rounds of "best remaining": highest score, then lowest page */
                for (int k = 0; k < topk; ++k) {
                    int best = -1;
                    for (int p = 0; p < wp; ++p) {
                        if (take[p])
                            continue;
                        if (best < 0 || s[p] > s[best])
                            best = p;
                    }
                    take[best] = 1;
                }
            }
            int32_t *out = sel + ((int64_t)b * Hk + kvh) * pt_stride;
            int n = 0;
            for (int p = 0; p < np; ++p)
                if (take[p])
                    out[n++] = p;
            nsel[(int64_t)b * Hk + kvh] = n;
        }
    }
    free(take);
}

/* Attention of every query head over the tokens of its kv head's chosen pages (sel /
 * nsel as from oracle_sparse_select), in fp64.  out [B][Hq][D], lse [B][Hq]. */
void oracle_sparse_decode(const uint16_t *q, const uint16_t *k_pages, const uint16_t *v_pages,
                          const int32_t *page_table, int pt_stride, const int32_t *seq_lens,
                          int B, int Hq, int Hk, int D, int P, double scale, const int32_t *sel,
                          const int32_t *nsel, double *out, double *lse)
{
    int g = Hq / Hk;
    int max_L = 0;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] > max_L)
            max_L = seq_lens[b];
#pragma omp parallel
    {
        double *K = (double *)malloc(sizeof(double) * ((size_t)max_L * D + 1));
        double *V = (double *)malloc(sizeof(double) * ((size_t)max_L * D + 1));
        double *s = (double *)malloc(sizeof(double) * ((size_t)max_L + 1));
        double *qd = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for collapse(2) schedule(dynamic)
        for (int b = 0; b < B; ++b)
            for (int kvh = 0; kvh < Hk; ++kvh) {
                int L = seq_lens[b];
                const int32_t *ps = sel + ((int64_t)b * Hk + kvh) * pt_stride;
                int n = 0; /* tokens gathered */
                for (int i = 0; i < nsel[(int64_t)b * Hk + kvh]; ++i) {
                    int p = ps[i];
                    int64_t phys = page_table[(int64_t)b * pt_stride + p];
                    int cnt = L - p * P < P ? L - p * P : P;
                    for (int t = 0; t < cnt; ++t, ++n)
                        for (int d = 0; d < D; ++d) {
                            K[(int64_t)n * D + d] = kv_value(k_pages, 0, NULL, Hk, P, D, phys, kvh, t, d);
                            V[(int64_t)n * D + d] = kv_value(v_pages, 0, NULL, Hk, P, D, phys, kvh, t, d);
                        }
                }
                for (int j = 0; j < g; ++j) {
                    int h = kvh * g + j;
                    for (int d = 0; d < D; ++d)
                        qd[d] = oracle_bf16_to_f64(q[((int64_t)b * Hq + h) * D + d]);
                    attend_row(qd, K, V, 0, n, D, scale, s, out + ((int64_t)b * Hq + h) * D,
                               lse + (int64_t)b * Hq + h);
                }
            }
        free(K);
        free(V);
        free(s);
        free(qd);
    }
}
