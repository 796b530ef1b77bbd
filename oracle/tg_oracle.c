/*
 * CPU ORACLE for ragged / prefix-shared / tiered paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's CPU-baseline leg
 * and reference arm may load this library. The product path (the CUDA library and its Python binding) never
 * calls it, and the two share no code: no headers, helpers, tables or constants.
 *
 * Plain, slow and written to be checked by eye: straight loops in the order the sources
 * describe, fp64 arithmetic for attention, no blocking, fusion or reordering. Where a
 * floating-point value decides an integer (the INT8 codes), the decision is taken in fp32,
 * the precision in which the stored scale is defined.
 *
 * Sources (web pages; cited by title and section):
 *  [Tangram]  "Tangram：为多轮 LLM Serving 解锁非均匀 KV Cache 压缩" (explainer of arXiv
 *             2606.06302), sections 核心方法 (关键发现; 三大机制 1 Budget Reservation,
 *             2 Ragged Paging, 3 Ahead-of-Time Load Balancing).
 *  [TTKV]     "TTKV: Temporal-Tiered KV Cache for Long-Context LLM Inference" (explainer of
 *             arXiv 2604.19769), 核心方法 1 Tier Layout, 2 Tier Content, 3 Tier Interaction.
 *  [CAP]      "面向 LLM 服务的 CAP 原则：长上下文大语言模型服务综述" (arXiv 2405.11299),
 *             §2.4.3 分布式加速, "加速单个请求" (online normaliser) and Fig. 5 (Dist Attention).
 *  [Radix]    "RadixAttention and KV reuse" lesson (Phase 17 · 06), section on the radix tree
 *             as KV index and its worked example tree.
 *  [SplitZip] "SplitZip: Ultra Fast Lossless KV Compression for Disaggregated LLM Serving"
 *             (explainer of arXiv 2605.01708), "Die SplitZip-Strategie", "Warum es schnell ist".
 *
 * Functions whose parity is pinned, and by what, are listed in the test suite
 * (tests/test_oracle_pins.py); none of the functions here is unpinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------------------------------
 * Small helpers (local to the oracle).
 * ------------------------------------------------------------------------------------- */

/* bf16 bits -> double, exactly (bf16 is the top half of an IEEE float32). */
static double or_bf16(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static int64_t or_ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int or_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------------------------------
 * Budget table -> retained length.
 * [Tangram] 关键发现: an input-invariant head ranking and a narrowly bounded per-head ratio
 * give a budget table; 三大机制 1 fixes each head's post-compression footprint at admission.
 * The page does not give the rounding; the reading used: ratio in parts per million,
 * round half up, at least one token, at most the full context, zero for an empty context.
 * ------------------------------------------------------------------------------------- */
void or_retained_lengths(int64_t n, const int32_t *full_len, const int32_t *ratio_ppm,
                         int32_t *kv_len) {
    for (int64_t i = 0; i < n; ++i) {
        int64_t L = full_len[i];
        if (L <= 0) {
            kv_len[i] = 0;
            continue;
        }
        int64_t r = ((int64_t)ratio_ppm[i] * L + 500000) / 1000000;
        if (r < 1) r = 1;
        if (r > L) r = L;
        kv_len[i] = (int32_t)r;
    }
}

/* ---------------------------------------------------------------------------------------
 * Budget groups. [Tangram] 三大机制 2 (Ragged Paging): heads with similar budgets go into
 * one group that has its own page table. Reading used: equal-count quantiles of the heads
 * ranked by budget (ascending budget, ties by index); position p of n -> group p*G/n.
 * ------------------------------------------------------------------------------------- */
void or_budget_groups(int32_t n, const int32_t *budget_ppm, int32_t n_groups, int32_t *group) {
    for (int32_t i = 0; i < n; ++i) {
        int64_t pos = 0;
        for (int32_t j = 0; j < n; ++j)
            if (budget_ppm[j] < budget_ppm[i] || (budget_ppm[j] == budget_ppm[i] && j < i)) ++pos;
        group[i] = (int32_t)(pos * n_groups / n);
    }
}

/* ---------------------------------------------------------------------------------------
 * Page layout of Budget Reservation, re-derived.
 * [Tangram] 三大机制 1: every (sequence, KV head) gets ceil(len/page) pages when its request
 * is admitted, once, so nothing is reclaimed while it runs.
 * [Radix] worked example: sequences that extend the same branch reuse its KV blocks; only
 * whole blocks are reused (the doc segment of 500 tokens counts 31 blocks).
 *
 * Free list: pages are taken from the front of free_order. Shared segments first, in segment
 * order, each segment: KV head ascending, page ascending, floor(tokens/page) pages per head.
 * Then sequences ascending; per sequence, KV head ascending: the head's page list is the
 * full pages of each of its prefix segments in chain order, followed by
 * ceil((kv_len - shared tokens)/page) private pages taken from the free list.
 *
 * seg_tokens[n_segs]; chain[n_seq][chain_len] segment ids, -1 = none (chain_len may be 0);
 * kv_len[n_seq][Hkv]. Output: page_ids, flat in (sequence, head, page) order (each head's
 * shared pages, then its private pages); head_count[n_seq][Hkv] gets each head's page
 * count. seg_pages_out[n_segs][Hkv][floor(seg_tokens/page)] flat, may be NULL.
 * Returns the number of page ids written, or -1 if the pool runs out, -2 if a head keeps
 * fewer tokens than its shared prefix.
 * ------------------------------------------------------------------------------------- */
int64_t or_reservation_layout(int64_t num_pages, const int32_t *free_order, int32_t page,
                              int32_t Hkv, int32_t n_segs, const int32_t *seg_tokens,
                              int32_t n_seq, int32_t chain_len, const int32_t *chain,
                              const int32_t *kv_len, int32_t *page_ids, int32_t *head_count,
                              int32_t *seg_pages_out) {
    int64_t next = 0; /* front of the free list */
    int64_t seg_total = 0;
    for (int32_t s = 0; s < n_segs; ++s) seg_total += (int64_t)Hkv * (seg_tokens[s] / page);
    int32_t *seg_pages = (int32_t *)malloc(sizeof(int32_t) * (size_t)(seg_total > 0 ? seg_total : 1));
    int64_t *seg_base = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_segs + 1));
    int64_t k = 0;
    for (int32_t s = 0; s < n_segs; ++s) {
        seg_base[s] = k;
        int32_t full = seg_tokens[s] / page;
        for (int32_t h = 0; h < Hkv; ++h)
            for (int32_t p = 0; p < full; ++p) {
                if (next >= num_pages) { free(seg_pages); free(seg_base); return -1; }
                seg_pages[k++] = free_order[next++];
            }
    }
    seg_base[n_segs] = k;
    if (seg_pages_out) memcpy(seg_pages_out, seg_pages, sizeof(int32_t) * (size_t)seg_total);

    int64_t w = 0;
    for (int32_t b = 0; b < n_seq; ++b) {
        for (int32_t h = 0; h < Hkv; ++h) {
            int64_t shared_tokens = 0;
            for (int32_t c = 0; c < chain_len; ++c) {
                int32_t s = chain[(int64_t)b * chain_len + c];
                if (s >= 0) shared_tokens += (int64_t)(seg_tokens[s] / page) * page;
            }
            int64_t n = kv_len[(int64_t)b * Hkv + h];
            if (n < shared_tokens) { free(seg_pages); free(seg_base); return -2; }
            int64_t cnt = 0;
            for (int32_t c = 0; c < chain_len; ++c) {
                int32_t s = chain[(int64_t)b * chain_len + c];
                if (s < 0) continue;
                int32_t full = seg_tokens[s] / page;
                for (int32_t p = 0; p < full; ++p)
                    page_ids[w++] = seg_pages[seg_base[s] + (int64_t)h * full + p];
                cnt += full;
            }
            int64_t priv = or_ceil_div(n - shared_tokens, page);
            for (int64_t p = 0; p < priv; ++p) {
                if (next >= num_pages) { free(seg_pages); free(seg_base); return -1; }
                page_ids[w++] = free_order[next++];
            }
            head_count[(int64_t)b * Hkv + h] = (int32_t)(cnt + priv);
        }
    }
    free(seg_pages);
    free(seg_base);
    return w;
}

/* ---------------------------------------------------------------------------------------
 * Group page tables. [Tangram] 三大机制 2 (Ragged Paging): one independent page table per
 * budget group. Layout used: group g's table is dense [B][H_g][P_g], heads of g in
 * ascending order, P_g = the largest page count among g's rows, unused slots = -1; the
 * group tables are concatenated in group order. head_off[b][h] = start of row (b, h).
 * page_ids/head_count as produced by or_reservation_layout.
 * group_off[G+1] gets each group table's start; returns the total table length.
 * ------------------------------------------------------------------------------------- */
int64_t or_group_tables(int32_t B, int32_t Hkv, const int32_t *group_of_head, int32_t n_groups,
                        const int32_t *page_ids, const int32_t *head_count, int32_t *table,
                        int64_t *head_off, int64_t *group_off) {
    /* start of each (b, h) in page_ids */
    int64_t *src = (int64_t *)malloc(sizeof(int64_t) * (size_t)B * Hkv + 8);
    int64_t acc = 0;
    for (int64_t i = 0; i < (int64_t)B * Hkv; ++i) { src[i] = acc; acc += head_count[i]; }

    int64_t pos = 0;
    for (int32_t g = 0; g < n_groups; ++g) {
        group_off[g] = pos;
        int32_t Hg = 0;
        int64_t Pg = 0;
        for (int32_t h = 0; h < Hkv; ++h) {
            if (group_of_head[h] != g) continue;
            ++Hg;
            for (int32_t b = 0; b < B; ++b)
                if (head_count[(int64_t)b * Hkv + h] > Pg) Pg = head_count[(int64_t)b * Hkv + h];
        }
        for (int32_t b = 0; b < B; ++b) {
            int32_t j = 0;
            for (int32_t h = 0; h < Hkv; ++h) {
                if (group_of_head[h] != g) continue;
                int64_t row = pos + ((int64_t)b * Hg + j) * Pg;
                head_off[(int64_t)b * Hkv + h] = row;
                int64_t cnt = head_count[(int64_t)b * Hkv + h];
                for (int64_t p = 0; p < Pg; ++p)
                    table[row + p] = p < cnt ? page_ids[src[(int64_t)b * Hkv + h] + p] : -1;
                ++j;
            }
        }
        pos += (int64_t)B * Hg * Pg;
    }
    group_off[n_groups] = pos;
    free(src);
    return pos;
}

/* ---------------------------------------------------------------------------------------
 * Decode attention over a paged KV cache, fp64.
 *
 * For query row (b, hq), KV head h = hq / (Hq/Hkv) (contiguous GQA groups), n = kv_len[b][h].
 * The retained tokens t = 0..n-1 are gathered through the page table
 *     page = table[head_off[b][h] + t / page_size],  slot = t % page_size,
 * and with s_t = scale * q . K_t,  m = max s_t:
 *     lse = m + ln sum_t exp(s_t - m),     out = sum_t exp(s_t - lse) V_t.
 * This is softmax attention; [CAP] §2.4.3 "加速单个请求": the online normaliser computes
 * exactly this blockwise, so a split kernel must reproduce it. n = 0 gives out = 0,
 * lse = -inf.
 *
 * tok_lo/tok_hi (both NULL, or [B][Hkv]) restrict each head to tokens [lo, hi): the partial
 * result of one split, normalised over that range (used to pin the merge below).
 * sel (n_sel entries of b*Hq + hq; n_sel < 0 means all rows) picks the rows to compute;
 * out is [n_rows][D], lse [n_rows] in selection order.
 * Inputs are bf16 bit patterns widened exactly. Returns 0, or 3 on a page id outside
 * [0, num_pages), or 1 on a bad argument.
 * ------------------------------------------------------------------------------------- */
static int or_row(int32_t b, int32_t hq, int32_t Hq, int32_t Hkv, int32_t D, int32_t page,
                  const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                  int64_t num_pages, const int32_t *table, const int64_t *head_off,
                  const int32_t *kv_len, const int32_t *tok_lo, const int32_t *tok_hi,
                  double scale, double *out, double *lse) {
    int32_t G = Hq / Hkv;
    int32_t h = hq / G;
    int64_t bh = (int64_t)b * Hkv + h;
    int64_t n = kv_len[bh];
    int64_t lo = tok_lo ? tok_lo[bh] : 0, hi = tok_hi ? tok_hi[bh] : n;
    if (hi > n) hi = n;
    for (int32_t d = 0; d < D; ++d) out[d] = 0.0;
    if (hi <= lo) { *lse = -INFINITY; return 0; }
    const uint16_t *qr = q + ((int64_t)b * Hq + hq) * D;
    double *s = (double *)malloc(sizeof(double) * (size_t)(hi - lo));
    double m = -INFINITY;
    for (int64_t t = lo; t < hi; ++t) {
        int64_t pid = table[head_off[bh] + t / page];
        if (pid < 0 || pid >= num_pages) { free(s); return 3; }
        const uint16_t *kr = k_pool + (pid * page + t % page) * D;
        double dot = 0.0;
        for (int32_t d = 0; d < D; ++d) dot += or_bf16(qr[d]) * or_bf16(kr[d]);
        s[t - lo] = scale * dot;
        if (s[t - lo] > m) m = s[t - lo];
    }
    double sum = 0.0;
    for (int64_t t = lo; t < hi; ++t) sum += exp(s[t - lo] - m);
    double L = m + log(sum);
    for (int64_t t = lo; t < hi; ++t) {
        int64_t pid = table[head_off[bh] + t / page];
        const uint16_t *vr = v_pool + (pid * page + t % page) * D;
        double w = exp(s[t - lo] - L);
        for (int32_t d = 0; d < D; ++d) out[d] += w * or_bf16(vr[d]);
    }
    *lse = L;
    free(s);
    return 0;
}

int or_decode(int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t page, const uint16_t *q,
              const uint16_t *k_pool, const uint16_t *v_pool, int64_t num_pages,
              const int32_t *table, const int64_t *head_off, const int32_t *kv_len,
              const int32_t *tok_lo, const int32_t *tok_hi, double scale, int64_t n_sel,
              const int64_t *sel, double *out, double *lse) {
    if (Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || page <= 0) return 1;
    int64_t rows = n_sel < 0 ? (int64_t)B * Hq : n_sel;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t id = n_sel < 0 ? r : sel[r];
        int e = or_row((int32_t)(id / Hq), (int32_t)(id % Hq), Hq, Hkv, D, page, q, k_pool,
                       v_pool, num_pages, table, head_off, kv_len, tok_lo, tok_hi, scale,
                       out + r * D, lse + r);
        if (e) {
#pragma omp atomic write
            err = e;
        }
    }
    return err;
}

/* ---------------------------------------------------------------------------------------
 * Tiered decode, fp64. [TTKV] 核心方法 1 (Tier Layout) and 2 (Tier Content): the most recent
 * tokens stay in the fast tier at high precision, older tokens go to the slow tier quantised
 * (INT8 here); 3 (Tier Interaction): attention streams the slow tier block by block.
 * Readings used: per head, the slow tier holds tokens [0, n - f) and the fast tier tokens
 * [n - f, n), f = fast_len[b][h] (clamped to n); each tier has its own page table whose row
 * starts at slot 0. A slow token's row is K_t = code_t * scale_t (fp32 scale per token per
 * head, symmetric INT8), likewise V; fast rows are bf16. The attention over the union is
 * the same softmax as in or_decode.
 * ------------------------------------------------------------------------------------- */
static int or_tiered_row(int32_t b, int32_t hq, int32_t Hq, int32_t Hkv, int32_t D,
                         int32_t page, const uint16_t *q, const int8_t *k_q8,
                         const int8_t *v_q8, const float *k_scale, const float *v_scale,
                         int64_t num_slow, const int32_t *slow_table, const int64_t *slow_off,
                         const uint16_t *k_fast, const uint16_t *v_fast, int64_t num_fast,
                         const int32_t *fast_table, const int64_t *fast_off,
                         const int32_t *kv_len, const int32_t *fast_len, double scale,
                         double *out, double *lse) {
    int32_t G = Hq / Hkv;
    int32_t h = hq / G;
    int64_t bh = (int64_t)b * Hkv + h;
    int64_t n = kv_len[bh];
    int64_t f = fast_len[bh] < n ? fast_len[bh] : n;
    int64_t n_slow = n - f;
    for (int32_t d = 0; d < D; ++d) out[d] = 0.0;
    if (n <= 0) { *lse = -INFINITY; return 0; }
    const uint16_t *qr = q + ((int64_t)b * Hq + hq) * D;
    double *krow = (double *)malloc(sizeof(double) * (size_t)D * 2);
    double *vrow = krow + D;
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    double m = -INFINITY;
    int err = 0;
    /* pass 1: scores */
    for (int64_t t = 0; t < n && !err; ++t) {
        if (t < n_slow) {
            int64_t pid = slow_table[slow_off[bh] + t / page];
            if (pid < 0 || pid >= num_slow) { err = 3; break; }
            int64_t row = pid * page + t % page;
            for (int32_t d = 0; d < D; ++d) krow[d] = (double)k_q8[row * D + d] * (double)k_scale[row];
        } else {
            int64_t u = t - n_slow;
            int64_t pid = fast_table[fast_off[bh] + u / page];
            if (pid < 0 || pid >= num_fast) { err = 3; break; }
            int64_t row = pid * page + u % page;
            for (int32_t d = 0; d < D; ++d) krow[d] = or_bf16(k_fast[row * D + d]);
        }
        double dot = 0.0;
        for (int32_t d = 0; d < D; ++d) dot += or_bf16(qr[d]) * krow[d];
        s[t] = scale * dot;
        if (s[t] > m) m = s[t];
    }
    if (!err) {
        double sum = 0.0;
        for (int64_t t = 0; t < n; ++t) sum += exp(s[t] - m);
        double L = m + log(sum);
        for (int64_t t = 0; t < n; ++t) {
            if (t < n_slow) {
                int64_t pid = slow_table[slow_off[bh] + t / page];
                int64_t row = pid * page + t % page;
                for (int32_t d = 0; d < D; ++d) vrow[d] = (double)v_q8[row * D + d] * (double)v_scale[row];
            } else {
                int64_t u = t - n_slow;
                int64_t pid = fast_table[fast_off[bh] + u / page];
                int64_t row = pid * page + u % page;
                for (int32_t d = 0; d < D; ++d) vrow[d] = or_bf16(v_fast[row * D + d]);
            }
            double w = exp(s[t] - L);
            for (int32_t d = 0; d < D; ++d) out[d] += w * vrow[d];
        }
        *lse = L;
    }
    free(s);
    free(krow);
    return err;
}

int or_tiered_decode(int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t page,
                     const uint16_t *q, const int8_t *k_q8, const int8_t *v_q8,
                     const float *k_scale, const float *v_scale, int64_t num_slow,
                     const int32_t *slow_table, const int64_t *slow_off,
                     const uint16_t *k_fast, const uint16_t *v_fast, int64_t num_fast,
                     const int32_t *fast_table, const int64_t *fast_off,
                     const int32_t *kv_len, const int32_t *fast_len, double scale,
                     int64_t n_sel, const int64_t *sel, double *out, double *lse) {
    if (Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || page <= 0) return 1;
    int64_t rows = n_sel < 0 ? (int64_t)B * Hq : n_sel;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t id = n_sel < 0 ? r : sel[r];
        int e = or_tiered_row((int32_t)(id / Hq), (int32_t)(id % Hq), Hq, Hkv, D, page, q,
                              k_q8, v_q8, k_scale, v_scale, num_slow, slow_table, slow_off,
                              k_fast, v_fast, num_fast, fast_table, fast_off, kv_len,
                              fast_len, scale, out + r * D, lse + r);
        if (e) {
#pragma omp atomic write
            err = e;
        }
    }
    return err;
}

/* ---------------------------------------------------------------------------------------
 * Slow-tier INT8 quantisation. [TTKV] 核心方法 1/3: older tokens are stored quantised, with
 * block-level quantisation in the slow tier; the page leaves the exact scheme open. Reading
 * used: symmetric absmax per token per head, separately for K and V:
 *     amax = max_d |x_d|,  scale = amax / 127  (fp32),
 *     code_d = clamp(nearbyint(x_d / scale), -127, 127)  (fp32 quotient, ties to even),
 * and amax = 0 gives scale = 0, all codes 0. rows = tokens, each of D bf16 values.
 * ------------------------------------------------------------------------------------- */
void or_quantize_int8(int64_t rows, int32_t D, const uint16_t *src, int8_t *codes, float *scale) {
    for (int64_t r = 0; r < rows; ++r) {
        float amax = 0.0f;
        for (int32_t d = 0; d < D; ++d) {
            float x = (float)or_bf16(src[r * D + d]);
            float a = fabsf(x);
            if (a > amax) amax = a;
        }
        float sc = amax / 127.0f;
        scale[r] = sc;
        for (int32_t d = 0; d < D; ++d) {
            if (amax == 0.0f) { codes[r * D + d] = 0; continue; }
            float x = (float)or_bf16(src[r * D + d]);
            float c = nearbyintf(x / sc);
            if (c > 127.0f) c = 127.0f;
            if (c < -127.0f) c = -127.0f;
            codes[r * D + d] = (int8_t)c;
        }
    }
}

/* ---------------------------------------------------------------------------------------
 * Slow-tier INT4 quantisation. [TTKV] 核心方法 1 Tier Layout names INT8/INT4 for the slow
 * tier and leaves the scheme open. Reading used, the INT8 rule with 7 levels a side:
 *     amax = max_d |x_d|,  scale = amax / 7  (fp32),
 *     code_d = clamp(nearbyint(x_d / scale), -7, 7)  (fp32 quotient, ties to even),
 * amax = 0 gives scale = 0 and all codes 0. Storage: two codes per byte as offset-binary
 * nibbles u = code + 8; byte i (i < D/2) of a row holds d = i in its low nibble and
 * d = i + D/2 in its high nibble. packed: uint8 [rows][D/2].
 * ------------------------------------------------------------------------------------- */
void or_quantize_int4(int64_t rows, int32_t D, const uint16_t *src, uint8_t *packed, float *scale) {
    int8_t *c = (int8_t *)malloc((size_t)D);
    for (int64_t r = 0; r < rows; ++r) {
        float amax = 0.0f;
        for (int32_t d = 0; d < D; ++d) {
            float a = fabsf((float)or_bf16(src[r * D + d]));
            if (a > amax) amax = a;
        }
        float sc = amax / 7.0f;
        scale[r] = sc;
        for (int32_t d = 0; d < D; ++d) {
            if (amax == 0.0f) { c[d] = 0; continue; }
            float v = nearbyintf((float)or_bf16(src[r * D + d]) / sc);
            if (v > 7.0f) v = 7.0f;
            if (v < -7.0f) v = -7.0f;
            c[d] = (int8_t)v;
        }
        for (int32_t i = 0; i < D / 2; ++i)
            packed[r * (D / 2) + i] = (uint8_t)((c[i] + 8) | ((c[i + D / 2] + 8) << 4));
    }
    free(c);
}

/* The codes of packed INT4 rows (layout of or_quantize_int4): codes int8 [rows][D]. */
void or_unpack_int4(int64_t rows, int32_t D, const uint8_t *packed, int8_t *codes) {
    for (int64_t r = 0; r < rows; ++r)
        for (int32_t i = 0; i < D / 2; ++i) {
            uint8_t b = packed[r * (D / 2) + i];
            codes[r * D + i] = (int8_t)((b & 0xF) - 8);
            codes[r * D + i + D / 2] = (int8_t)((b >> 4) - 8);
        }
}

/* ---------------------------------------------------------------------------------------
 * Merge of split results. [CAP] §2.4.3 (online normaliser) and Fig. 5 (Dist Attention: the
 * decode query is one token and the partial results over disjoint KV ranges are combined).
 * For splits j = 0..S-1 with normalised partials o_j and log-sum-exp lse_j:
 *     lse = ln sum_j exp(lse_j),   out = sum_j exp(lse_j - lse) o_j,
 * summed in split order. Splits with lse_j = -inf contribute nothing; all -inf gives
 * out = 0, lse = -inf. parts_o [S][rows][D], parts_lse [S][rows].
 * ------------------------------------------------------------------------------------- */
void or_lse_merge(int32_t S, int64_t rows, int32_t D, const double *parts_o,
                  const double *parts_lse, double *out, double *lse) {
    for (int64_t r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int32_t j = 0; j < S; ++j)
            if (parts_lse[(int64_t)j * rows + r] > m) m = parts_lse[(int64_t)j * rows + r];
        for (int32_t d = 0; d < D; ++d) out[r * D + d] = 0.0;
        if (m == -INFINITY) { lse[r] = -INFINITY; continue; }
        double sum = 0.0;
        for (int32_t j = 0; j < S; ++j) sum += exp(parts_lse[(int64_t)j * rows + r] - m);
        double L = m + log(sum);
        for (int32_t j = 0; j < S; ++j) {
            double w = exp(parts_lse[(int64_t)j * rows + r] - L);
            for (int32_t d = 0; d < D; ++d) out[r * D + d] += w * parts_o[((int64_t)j * rows + r) * D + d];
        }
        lse[r] = L;
    }
}

/* ---------------------------------------------------------------------------------------
 * Ahead-of-time placement of sequences on GPUs. [Tangram] 三大机制 3: requests are
 * partitioned across GPUs ahead of time by the heads' total KV footprint. Reading used:
 * longest-processing-time greedy: sequences by bytes descending (ties by index), each to the
 * GPU with the least assigned bytes so far (ties by lowest GPU index).
 * ------------------------------------------------------------------------------------- */
void or_place_sequences(int32_t n_seq, const int64_t *seq_bytes, int32_t n_gpus, int32_t *gpu_of_seq) {
    int32_t *order = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_seq > 0 ? n_seq : 1));
    int64_t *load = (int64_t *)calloc((size_t)(n_gpus > 0 ? n_gpus : 1), sizeof(int64_t));
    for (int32_t i = 0; i < n_seq; ++i) order[i] = i;
    /* selection sort: plain and obviously correct */
    for (int32_t i = 0; i < n_seq; ++i) {
        int32_t best = i;
        for (int32_t j = i + 1; j < n_seq; ++j) {
            int32_t a = order[j], c = order[best];
            if (seq_bytes[a] > seq_bytes[c] || (seq_bytes[a] == seq_bytes[c] && a < c)) best = j;
        }
        int32_t t = order[i]; order[i] = order[best]; order[best] = t;
    }
    for (int32_t i = 0; i < n_seq; ++i) {
        int32_t g = 0;
        for (int32_t k = 1; k < n_gpus; ++k) if (load[k] < load[g]) g = k;
        gpu_of_seq[order[i]] = g;
        load[g] += seq_bytes[order[i]];
    }
    free(order);
    free(load);
}

/* ---------------------------------------------------------------------------------------
 * Decode-step write path: where the token of a new decode step goes in a head whose
 * footprint is fixed. [Tangram] 三大机制 1 (Budget Reservation): each head's post-compression
 * footprint is fixed when the request starts, so a decode step never reclaims or grows pages;
 * a head whose reserved slots are all in use replaces one retained token. Which one is the
 * compression algorithm's choice; Tangram plugs in H2O and others unchanged (落地形态). The
 * two rules below are the ones [CAP] §2.4.1 describes for decoder-only models:
 *  (3) static: LM-Infinite / StreamingLLM keep the first tokens and the last L tokens;
 *  (4) dynamic: H2O keeps the last L tokens plus the tokens with the largest attention
 *      accumulated at run time.
 * A head is described by its `budget` reserved slots, `kv_len` of them in use (slots
 * 0 .. kv_len-1), and slot_pos[i] = sequence position of the token in slot i.
 * ------------------------------------------------------------------------------------- */

/* Sink + recent. Readings used: the first s = min(sink, budget - 1) positions of the
 * sequence are the sinks; with a free slot the new token takes slot kv_len; otherwise it
 * replaces the oldest non-sink token (smallest position >= s), so that the head keeps
 * positions 0 .. s-1 and the budget - s most recent ones. Returns the slot, or -1 when
 * budget < 1. */
int32_t or_sink_recent_slot(int32_t budget, int32_t sink, int32_t kv_len, const int32_t *slot_pos) {
    if (budget < 1) return -1;
    if (kv_len < budget) return kv_len;
    int32_t s = sink < budget - 1 ? sink : budget - 1;
    if (s < 0) s = 0;
    int32_t best = -1;
    for (int32_t i = 0; i < kv_len; ++i) {
        if (slot_pos[i] < s) continue;
        if (best < 0 || slot_pos[i] < slot_pos[best]) best = i;
    }
    return best;
}

/* H2O. Readings used: the protected recent window is the last `recent` positions before the
 * new token (positions >= new_pos - recent); with a free slot the new token takes slot
 * kv_len; otherwise the victim is the slot with the lowest accumulated score among the older
 * tokens (ties: the lowest slot); if every token is recent, the slot of the oldest token.
 * The comparison is on the fp32 scores as stored. Returns the slot, or -1 when budget < 1. */
int32_t or_h2o_victim(int32_t budget, int32_t recent, int32_t kv_len, const int32_t *slot_pos,
                      const float *score, int32_t new_pos) {
    if (budget < 1) return -1;
    if (kv_len < budget) return kv_len;
    int32_t best = -1, oldest = 0;
    for (int32_t i = 0; i < kv_len; ++i) {
        if (slot_pos[i] < slot_pos[oldest]) oldest = i;
        if ((int64_t)slot_pos[i] >= (int64_t)new_pos - recent) continue;
        if (best < 0 || score[i] < score[best]) best = i;
    }
    return best >= 0 ? best : oldest;
}

/* Attention scores of every retained token, fp64: s[t][g] = scale * q[b][h*G+g] . K[t] for
 * the tokens of every (b, h), t < kv_len[b][h], gathered through the table as in or_decode.
 * Output out[(head_off[b][h] * page + t) * G + g]; slots beyond kv_len are left untouched.
 * Returns 0, 3 on a page id outside the pool, 1 on a bad argument. */
int or_token_scores(int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t page, const uint16_t *q,
                    const uint16_t *k_pool, int64_t num_pages, const int32_t *table,
                    const int64_t *head_off, const int32_t *kv_len, double scale, double *out) {
    if (Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || page <= 0) return 1;
    int32_t G = Hq / Hkv;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < (int64_t)B * Hkv; ++bh) {
        int32_t b = (int32_t)(bh / Hkv), h = (int32_t)(bh % Hkv);
        for (int64_t t = 0; t < kv_len[bh]; ++t) {
            int64_t pid = table[head_off[bh] + t / page];
            if (pid < 0 || pid >= num_pages) {
#pragma omp atomic write
                err = 3;
                break;
            }
            const uint16_t *kr = k_pool + (pid * page + t % page) * D;
            for (int32_t g = 0; g < G; ++g) {
                const uint16_t *qr = q + ((int64_t)b * Hq + (int64_t)h * G + g) * D;
                double dot = 0.0;
                for (int32_t d = 0; d < D; ++d) dot += or_bf16(qr[d]) * or_bf16(kr[d]);
                out[(head_off[bh] * page + t) * G + g] = scale * dot;
            }
        }
    }
    return err;
}

/* H2O accumulation for one head: each retained token's score grows by the attention the
 * current step's queries pay it, summed over the G query heads of the KV head:
 *     score[t] += sum_g exp(s[t][g] - lse[g]),
 * in fp64 from the fp32 score, rounded to fp32 once. s is [n][G], lse [G]. */
void or_h2o_accumulate(int32_t n, int32_t G, const double *s, const double *lse,
                       const float *score_in, float *score_out) {
    for (int32_t t = 0; t < n; ++t) {
        double acc = (double)score_in[t];
        for (int32_t g = 0; g < G; ++g) acc += exp(s[(int64_t)t * G + g] - lse[g]);
        score_out[t] = (float)acc;
    }
}

/* ---------------------------------------------------------------------------------------
 * Tier migration. [TTKV] 核心方法 1 (Tier Layout: recent tokens in the fast high-precision
 * tier, older ones in the slow quantised tier) and 2 (Tier Content: the most recent tokens, as
 * many as the fast tier holds, are fast; the rest slow). Readings used: the fast tier of a head
 * holds the last f <= cap tokens, the token at position p in fast slot p mod cap; the slow tier
 * holds positions [0, n - f) at slow index = position. Appending position n: with f < cap (only
 * when every token is fast, n == f) it takes fast slot n and nothing moves; with f == cap the
 * oldest fast token (position n - cap) moves to slow index n - cap (quantised by
 * or_quantize_int8) and the new token takes its slot. Returns 0 with the slots, or -1 when the
 * state is outside these rules or the slow tier has no reserved slot left.
 * ------------------------------------------------------------------------------------- */
int or_tier_step(int32_t n, int32_t f, int32_t cap, int32_t slow_cap, int32_t *fast_slot,
                 int32_t *slow_index) {
    *fast_slot = -1;
    *slow_index = -1;
    if (cap < 1 || f < 0 || f > cap || f > n) return -1;
    if (f < cap) {
        if (n != f) return -1;
        *fast_slot = n;
        return 0;
    }
    int32_t old = n - cap;
    if (old >= slow_cap) return -1;
    *slow_index = old;
    *fast_slot = old % cap;
    return 0;
}

/* ---------------------------------------------------------------------------------------
 * SplitZip: lossless BF16 codec for KV transfer. [SplitZip] explainer (arXiv 2605.01708),
 * "Die SplitZip-Strategie" and "Warum es schnell ist": a bf16 value is sign, 8-bit exponent and
 * 7-bit mantissa; exponents repeat, so the 16 most frequent get 4-bit codes (two per byte), the
 * rare ones go to an escape stream (position, exponent) that decoding applies as overwrites.
 * Readings used: the codebook lists 16 exponents by count descending, ties by exponent
 * ascending, over all 256 exponent values (so it always holds 16 distinct entries); sign and
 * mantissa are stored as one byte per element, (sign << 7) | mantissa; the 4-bit code of
 * element i sits in byte i/2, low nibble for even i; an escaped element carries code 0; escapes
 * are listed in ascending position.
 * ------------------------------------------------------------------------------------- */
void or_splitzip_codebook(int64_t n, const uint16_t *x, uint8_t *codebook) {
    int64_t count[256];
    for (int e = 0; e < 256; ++e) count[e] = 0;
    for (int64_t i = 0; i < n; ++i) ++count[(x[i] >> 7) & 0xFF];
    int taken[256];
    for (int e = 0; e < 256; ++e) taken[e] = 0;
    for (int k = 0; k < 16; ++k) {
        int best = -1;
        for (int e = 0; e < 256; ++e) {
            if (taken[e]) continue;
            if (best < 0 || count[e] > count[best]) best = e;  /* ties keep the smaller exponent */
        }
        taken[best] = 1;
        codebook[k] = (uint8_t)best;
    }
}

int64_t or_splitzip_encode(int64_t n, const uint16_t *x, const uint8_t *codebook, uint8_t *sm,
                           uint8_t *codes, int64_t *esc_pos, uint8_t *esc_exp) {
    int64_t n_esc = 0;
    for (int64_t i = 0; i < (n + 1) / 2; ++i) codes[i] = 0;
    for (int64_t i = 0; i < n; ++i) {
        int sign = (x[i] >> 15) & 1, e = (x[i] >> 7) & 0xFF, m = x[i] & 0x7F;
        sm[i] = (uint8_t)((sign << 7) | m);
        int code = -1;
        for (int k = 0; k < 16; ++k)
            if (codebook[k] == e) code = k;
        if (code < 0) {
            esc_pos[n_esc] = i;
            esc_exp[n_esc] = (uint8_t)e;
            ++n_esc;
            code = 0;
        }
        codes[i / 2] |= (uint8_t)(code << (4 * (i % 2)));
    }
    return n_esc;
}

void or_splitzip_decode(int64_t n, const uint8_t *codebook, const uint8_t *sm, const uint8_t *codes,
                        int64_t n_esc, const int64_t *esc_pos, const uint8_t *esc_exp, uint16_t *x) {
    for (int64_t i = 0; i < n; ++i) {
        int code = (codes[i / 2] >> (4 * (i % 2))) & 0xF;
        int e = codebook[code];
        x[i] = (uint16_t)(((sm[i] >> 7) << 15) | (e << 7) | (sm[i] & 0x7F));
    }
    for (int64_t j = 0; j < n_esc; ++j) {
        int64_t i = esc_pos[j];
        x[i] = (uint16_t)((x[i] & 0x807F) | (esc_exp[j] << 7));
    }
}
