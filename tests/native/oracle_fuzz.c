/* Memory-safety drive of the CPU oracle (oracle/tg_oracle.c), built with AddressSanitizer and
 * UndefinedBehaviorSanitizer by tests/test_host_sanitizers.py and run on seeded random cases:
 * every exported function, on shapes from one token to a few pages per head, with shared
 * prefixes, empty heads, splits, both slow-tier widths, the write-path rules and the codec.
 * The checks are the ones any correct result meets (ranges, convex combinations, a merge of
 * splits equal to the unsplit result, lossless round trips); the values themselves are pinned
 * elsewhere. Any sanitizer report ends the run with a non-zero status. No GPU involved. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

/* the oracle's entry points (it ships no header of its own) */
void or_retained_lengths(int64_t n, const int32_t *full_len, const int32_t *ratio_ppm, int32_t *kv_len);
void or_budget_groups(int32_t n, const int32_t *budget_ppm, int32_t n_groups, int32_t *group);
int64_t or_reservation_layout(int64_t num_pages, const int32_t *free_order, int32_t page, int32_t Hkv,
                              int32_t n_segs, const int32_t *seg_tokens, int32_t n_seq, int32_t chain_len,
                              const int32_t *chain, const int32_t *kv_len, int32_t *page_ids,
                              int32_t *head_count, int32_t *seg_pages_out);
int64_t or_group_tables(int32_t B, int32_t Hkv, const int32_t *group_of_head, int32_t n_groups,
                        const int32_t *page_ids, const int32_t *head_count, int32_t *table,
                        int64_t *head_off, int64_t *group_off);
int or_decode(int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t page, const uint16_t *q,
              const uint16_t *k_pool, const uint16_t *v_pool, int64_t num_pages, const int32_t *table,
              const int64_t *head_off, const int32_t *kv_len, const int32_t *tok_lo, const int32_t *tok_hi,
              double scale, int64_t n_sel, const int64_t *sel, double *out, double *lse);
int or_tiered_decode(int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t page, const uint16_t *q,
                     const int8_t *k_q8, const int8_t *v_q8, const float *k_scale, const float *v_scale,
                     int64_t num_slow, const int32_t *slow_table, const int64_t *slow_off,
                     const uint16_t *k_fast, const uint16_t *v_fast, int64_t num_fast,
                     const int32_t *fast_table, const int64_t *fast_off, const int32_t *kv_len,
                     const int32_t *fast_len, double scale, int64_t n_sel, const int64_t *sel, double *out,
                     double *lse);
void or_quantize_int8(int64_t rows, int32_t D, const uint16_t *src, int8_t *codes, float *scale);
void or_quantize_int4(int64_t rows, int32_t D, const uint16_t *src, uint8_t *packed, float *scale);
void or_unpack_int4(int64_t rows, int32_t D, const uint8_t *packed, int8_t *codes);
void or_lse_merge(int32_t S, int64_t rows, int32_t D, const double *parts_o, const double *parts_lse,
                  double *out, double *lse);
void or_place_sequences(int32_t n_seq, const int64_t *seq_bytes, int32_t n_gpus, int32_t *gpu_of_seq);
int32_t or_sink_recent_slot(int32_t budget, int32_t sink, int32_t kv_len, const int32_t *slot_pos);
int32_t or_h2o_victim(int32_t budget, int32_t recent, int32_t kv_len, const int32_t *slot_pos,
                      const float *score, int32_t new_pos);
int or_token_scores(int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t page, const uint16_t *q,
                    const uint16_t *k_pool, int64_t num_pages, const int32_t *table, const int64_t *head_off,
                    const int32_t *kv_len, double scale, double *out);
void or_h2o_accumulate(int32_t n, int32_t G, const double *s, const double *lse, const float *score_in,
                       float *score_out);
int or_tier_step(int32_t n, int32_t f, int32_t cap, int32_t slow_cap, int32_t *fast_slot, int32_t *slow_index);
void or_splitzip_codebook(int64_t n, const uint16_t *x, uint8_t *codebook);
int64_t or_splitzip_encode(int64_t n, const uint16_t *x, const uint8_t *codebook, uint8_t *sm, uint8_t *codes,
                           int64_t *esc_pos, uint8_t *esc_exp);
void or_splitzip_decode(int64_t n, const uint8_t *codebook, const uint8_t *sm, const uint8_t *codes,
                        int64_t n_esc, const int64_t *esc_pos, const uint8_t *esc_exp, uint16_t *x);

#define CHECK(c)                                                              \
    do {                                                                      \
        if (!(c)) {                                                           \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c);   \
            exit(2);                                                          \
        }                                                                     \
    } while (0)

static uint64_t g_state = 0x5EED0F0ACE5ULL;
static uint64_t next_u64(void) { /* SplitMix64 (Steele, Lea & Flood 2014), the driver's own draws */
    uint64_t z = (g_state += 0x9E3779B97F4A7C15ULL);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}
static int64_t uni(int64_t lo, int64_t hi) { return lo + (int64_t)(next_u64() % (uint64_t)(hi - lo + 1)); }
static uint16_t bf16_bits(double x) { /* truncation to bf16: any finite bf16 pattern will do here */
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}
static double bf16_val(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}
static double normal(void) {
    double u1 = ((next_u64() >> 11) + 1.0) / 9007199254740993.0, u2 = (next_u64() >> 11) / 9007199254740992.0;
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}
static void *xcalloc(size_t n, size_t sz) {
    void *p = calloc(n ? n : 1, sz);
    CHECK(p);
    return p;
}

static void round_case(void) {
    const int32_t page = 16;
    const int32_t B = (int32_t)uni(1, 4), Hkv = (int32_t)uni(1, 4), G = 1 << uni(0, 2), Hq = Hkv * G;
    const int32_t D = uni(0, 1) ? 64 : 32;
    const int64_t BH = (int64_t)B * Hkv;

    /* admission: lengths, groups */
    int32_t *full = xcalloc((size_t)BH, 4), *ratio = xcalloc((size_t)BH, 4), *kv = xcalloc((size_t)BH, 4);
    for (int64_t i = 0; i < BH; ++i) {
        full[i] = (int32_t)uni(0, 90);
        ratio[i] = (int32_t)uni(0, 1000000);
    }
    or_retained_lengths(BH, full, ratio, kv);
    for (int64_t i = 0; i < BH; ++i) CHECK(kv[i] >= 0 && kv[i] <= full[i] && (full[i] == 0 || kv[i] >= 1));
    const int32_t n_groups = (int32_t)uni(1, Hkv);
    int32_t *budget = xcalloc((size_t)Hkv, 4), *goh = xcalloc((size_t)Hkv, 4);
    for (int32_t h = 0; h < Hkv; ++h) budget[h] = (int32_t)uni(0, 1000000);
    or_budget_groups(Hkv, budget, n_groups, goh);
    for (int32_t h = 0; h < Hkv; ++h) CHECK(goh[h] >= 0 && goh[h] < n_groups);

    /* reservation with one optional shared segment per sequence */
    const int32_t seg_tokens[1] = {(int32_t)uni(0, 40)};
    const int32_t shared = seg_tokens[0] / page * page;
    int32_t *chain = xcalloc((size_t)B, 4);
    for (int32_t b = 0; b < B; ++b) {
        chain[b] = uni(0, 1) ? 0 : -1;
        if (chain[b] == 0)
            for (int32_t h = 0; h < Hkv; ++h)
                if (kv[(int64_t)b * Hkv + h] < shared) kv[(int64_t)b * Hkv + h] = shared;
    }
    int64_t need = (int64_t)Hkv * (seg_tokens[0] / page);
    for (int64_t i = 0; i < BH; ++i) need += (kv[i] + page - 1) / page;
    const int64_t num_pages = need + uni(0, 5);
    int32_t *order = xcalloc((size_t)num_pages, 4);
    for (int64_t i = 0; i < num_pages; ++i) order[i] = (int32_t)i;
    for (int64_t i = num_pages - 1; i > 0; --i) {
        int64_t j = uni(0, i);
        int32_t t = order[i];
        order[i] = order[j];
        order[j] = t;
    }
    int32_t *ids = xcalloc((size_t)(need + 1) * 2, 4), *count = xcalloc((size_t)BH, 4);
    int32_t *segp = xcalloc((size_t)Hkv * 4, 4);
    const int64_t w = or_reservation_layout(num_pages, order, page, Hkv, 1, seg_tokens, B, 1, chain, kv, ids,
                                            count, segp);
    CHECK(w >= 0);
    int64_t total = 0;
    for (int64_t i = 0; i < BH; ++i) total += count[i];
    CHECK(total == w);
    /* exactly the pages the layout takes: a pool one page short is refused */
    int64_t exact = (int64_t)Hkv * (seg_tokens[0] / page);
    for (int32_t b = 0; b < B; ++b)
        for (int32_t h = 0; h < Hkv; ++h)
            exact += (kv[(int64_t)b * Hkv + h] - (chain[b] == 0 ? shared : 0) + page - 1) / page;
    if (exact > 0)
        CHECK(or_reservation_layout(exact - 1, order, page, Hkv, 1, seg_tokens, B, 1, chain, kv, ids, count,
                                    NULL) == -1);
    CHECK(or_reservation_layout(exact, order, page, Hkv, 1, seg_tokens, B, 1, chain, kv, ids, count, segp) == w);

    /* group tables */
    int64_t *goff = xcalloc((size_t)n_groups + 1, 8), *hoff = xcalloc((size_t)BH, 8);
    int64_t tmax = 0;
    for (int32_t g = 0; g < n_groups; ++g) {
        int64_t hg = 0, pg = 0;
        for (int32_t h = 0; h < Hkv; ++h)
            if (goh[h] == g) {
                ++hg;
                for (int32_t b = 0; b < B; ++b)
                    if (count[(int64_t)b * Hkv + h] > pg) pg = count[(int64_t)b * Hkv + h];
            }
        tmax += (int64_t)B * hg * pg;
    }
    int32_t *table = xcalloc((size_t)tmax + 1, 4);
    CHECK(or_group_tables(B, Hkv, goh, n_groups, ids, count, table, hoff, goff) == tmax);
    for (int64_t i = 0; i < BH; ++i)
        for (int32_t p = 0; p < count[i]; ++p) CHECK(table[hoff[i] + p] >= 0 && table[hoff[i] + p] < num_pages);

    /* decode: all rows, a selection, two splits merged */
    uint16_t *kp = xcalloc((size_t)num_pages * page * D, 2), *vp = xcalloc((size_t)num_pages * page * D, 2);
    uint16_t *q = xcalloc((size_t)B * Hq * D, 2);
    double vmax = 0.0;
    for (int64_t i = 0; i < num_pages * page * D; ++i) {
        kp[i] = bf16_bits(normal());
        vp[i] = bf16_bits(normal());
        if (fabs(bf16_val(vp[i])) > vmax) vmax = fabs(bf16_val(vp[i]));
    }
    for (int64_t i = 0; i < (int64_t)B * Hq * D; ++i) q[i] = bf16_bits(normal());
    const int64_t rows = (int64_t)B * Hq;
    double *out = xcalloc((size_t)rows * D, 8), *lse = xcalloc((size_t)rows, 8);
    const double scale = 1.0 / sqrt((double)D);
    CHECK(or_decode(B, Hq, Hkv, D, page, q, kp, vp, num_pages, table, hoff, kv, NULL, NULL, scale, -1, NULL, out,
                    lse) == 0);
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t bh = (r / Hq) * Hkv + (r % Hq) / G;
        if (kv[bh] == 0) {
            CHECK(isinf(lse[r]) && lse[r] < 0);
            for (int32_t d = 0; d < D; ++d) CHECK(out[r * D + d] == 0.0);
        } else {
            CHECK(isfinite(lse[r]));
            for (int32_t d = 0; d < D; ++d) CHECK(fabs(out[r * D + d]) <= vmax * (1 + 1e-12));
        }
    }
    int64_t sel[2] = {uni(0, rows - 1), uni(0, rows - 1)};
    double out2[2 * 64], lse2[2];
    CHECK(or_decode(B, Hq, Hkv, D, page, q, kp, vp, num_pages, table, hoff, kv, NULL, NULL, scale, 2, sel, out2,
                    lse2) == 0);
    for (int k = 0; k < 2; ++k) {
        CHECK(lse2[k] == lse[sel[k]] || (isinf(lse2[k]) && isinf(lse[sel[k]])));
        for (int32_t d = 0; d < D; ++d) CHECK(out2[k * D + d] == out[sel[k] * D + d]);
    }
    int32_t *lo = xcalloc((size_t)BH, 4), *mid = xcalloc((size_t)BH, 4), *hi = xcalloc((size_t)BH, 4);
    for (int64_t i = 0; i < BH; ++i) {
        mid[i] = (int32_t)uni(0, kv[i]);
        hi[i] = kv[i];
    }
    double *po = xcalloc((size_t)2 * rows * D, 8), *pl = xcalloc((size_t)2 * rows, 8);
    CHECK(or_decode(B, Hq, Hkv, D, page, q, kp, vp, num_pages, table, hoff, kv, lo, mid, scale, -1, NULL, po,
                    pl) == 0);
    CHECK(or_decode(B, Hq, Hkv, D, page, q, kp, vp, num_pages, table, hoff, kv, mid, hi, scale, -1, NULL,
                    po + rows * D, pl + rows) == 0);
    double *mo = xcalloc((size_t)rows * D, 8), *ml = xcalloc((size_t)rows, 8);
    or_lse_merge(2, rows, D, po, pl, mo, ml);
    for (int64_t r = 0; r < rows; ++r) {
        CHECK((isinf(ml[r]) && isinf(lse[r])) || fabs(ml[r] - lse[r]) <= 1e-9);
        for (int32_t d = 0; d < D; ++d) CHECK(fabs(mo[r * D + d] - out[r * D + d]) <= 1e-9);
    }
    /* a page id outside the pool is reported, not read */
    if (tmax > 0 && count[0] > 0) {
        const int32_t keep = table[hoff[0]];
        table[hoff[0]] = (int32_t)num_pages;
        CHECK(or_decode(B, Hq, Hkv, D, page, q, kp, vp, num_pages, table, hoff, kv, NULL, NULL, scale, -1, NULL,
                        out, lse) == 3);
        table[hoff[0]] = keep;
    }

    /* token scores and H2O accumulation */
    double *sc = xcalloc((size_t)(tmax + 1) * page * G, 8);
    CHECK(or_token_scores(B, Hq, Hkv, D, page, q, kp, num_pages, table, hoff, kv, scale, sc) == 0);
    {
        const int32_t n = kv[0];
        double *s0 = xcalloc((size_t)n * G + 1, 8), lse0[8];
        float *si = xcalloc((size_t)n + 1, 4), *so = xcalloc((size_t)n + 1, 4);
        for (int32_t t = 0; t < n; ++t)
            for (int32_t g = 0; g < G; ++g) s0[(int64_t)t * G + g] = sc[(hoff[0] * page + t) * G + g];
        CHECK(or_decode(B, Hq, Hkv, D, page, q, kp, vp, num_pages, table, hoff, kv, NULL, NULL, scale, -1, NULL,
                        out, lse) == 0);
        for (int32_t g = 0; g < G; ++g) lse0[g] = lse[g];
        for (int32_t t = 0; t < n; ++t) si[t] = (float)uni(0, 100);
        or_h2o_accumulate(n, G, s0, lse0, si, so);
        double added = 0.0;
        for (int32_t t = 0; t < n; ++t) {
            CHECK(so[t] >= si[t]);
            added += (double)so[t] - (double)si[t];
        }
        CHECK(n == 0 || fabs(added - G) <= 1e-3 * G + 1e-4 * n);
        free(s0);
        free(si);
        free(so);
    }

    /* tiered: the same tokens, the older part of every head quantised (INT8, then INT4) */
    int32_t *fl = xcalloc((size_t)BH, 4);
    for (int64_t i = 0; i < BH; ++i) fl[i] = (int32_t)uni(0, kv[i] + 3);
    const int64_t prow = num_pages * page;
    int8_t *kq = xcalloc((size_t)prow * D, 1), *vq = xcalloc((size_t)prow * D, 1);
    float *ks = xcalloc((size_t)prow, 4), *vs = xcalloc((size_t)prow, 4);
    or_quantize_int8(prow, D, kp, kq, ks);
    or_quantize_int8(prow, D, vp, vq, vs);
    for (int64_t i = 0; i < prow * D; ++i) CHECK(kq[i] >= -127 && kq[i] <= 127);
    CHECK(or_tiered_decode(B, Hq, Hkv, D, page, q, kq, vq, ks, vs, num_pages, table, hoff, kp, vp, num_pages, table,
                           hoff, kv, fl, scale, -1, NULL, out, lse) == 0);
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t bh = (r / Hq) * Hkv + (r % Hq) / G;
        CHECK(kv[bh] == 0 ? (isinf(lse[r]) && lse[r] < 0) : isfinite(lse[r]));
    }
    uint8_t *k4 = xcalloc((size_t)prow * D / 2, 1), *v4 = xcalloc((size_t)prow * D / 2, 1);
    or_quantize_int4(prow, D, kp, k4, ks);
    or_quantize_int4(prow, D, vp, v4, vs);
    or_unpack_int4(prow, D, k4, kq);
    or_unpack_int4(prow, D, v4, vq);
    for (int64_t i = 0; i < prow * D; ++i) CHECK(kq[i] >= -7 && kq[i] <= 7 && vq[i] >= -7 && vq[i] <= 7);
    CHECK(or_tiered_decode(B, Hq, Hkv, D, page, q, kq, vq, ks, vs, num_pages, table, hoff, kp, vp, num_pages, table,
                           hoff, kv, fl, scale, -1, NULL, out, lse) == 0);

    /* placement, write-path rules, tier steps */
    int64_t *bytes = xcalloc((size_t)B, 8);
    int32_t *gpu = xcalloc((size_t)B, 4);
    for (int32_t b = 0; b < B; ++b) bytes[b] = uni(0, 1 << 20);
    const int32_t n_gpus = (int32_t)uni(1, 5);
    or_place_sequences(B, bytes, n_gpus, gpu);
    for (int32_t b = 0; b < B; ++b) CHECK(gpu[b] >= 0 && gpu[b] < n_gpus);
    {
        const int32_t budget_slots = (int32_t)uni(1, 12), used = (int32_t)uni(0, budget_slots);
        int32_t pos[12];
        float score[12];
        for (int32_t i = 0; i < used; ++i) {
            pos[i] = i * 2 + (int32_t)uni(0, 1);
            score[i] = (float)uni(0, 50);
        }
        const int32_t s1 = or_sink_recent_slot(budget_slots, (int32_t)uni(0, 14), used, pos);
        CHECK(s1 >= 0 && s1 < budget_slots);
        const int32_t s2 = or_h2o_victim(budget_slots, (int32_t)uni(0, 14), used, pos, score, 2 * used + 2);
        CHECK(s2 >= 0 && s2 < budget_slots);
        CHECK(or_sink_recent_slot(0, 1, 0, pos) == -1 && or_h2o_victim(0, 1, 0, pos, score, 0) == -1);
    }
    {
        const int32_t cap = (int32_t)uni(1, 20), slow_cap = (int32_t)uni(0, 40);
        int32_t n = 0, f = 0, fs, si;
        while (or_tier_step(n, f, cap, slow_cap, &fs, &si) == 0) {
            CHECK(fs >= 0 && fs < cap && si < slow_cap);
            ++n;
            if (f < cap) ++f;
            CHECK(n < 100);
        }
        CHECK(n == cap + slow_cap);
    }

    /* SplitZip round trip on any bit patterns */
    {
        const int64_t n = uni(0, 300);
        uint16_t *x = xcalloc((size_t)n, 2), *y = xcalloc((size_t)n, 2);
        for (int64_t i = 0; i < n; ++i) x[i] = uni(0, 3) ? bf16_bits(normal()) : (uint16_t)next_u64();
        uint8_t cb[16], *sm = xcalloc((size_t)n, 1), *codes = xcalloc((size_t)(n + 1) / 2, 1);
        int64_t *ep = xcalloc((size_t)n, 8);
        uint8_t *ee = xcalloc((size_t)n, 1);
        or_splitzip_codebook(n, x, cb);
        const int64_t ne = or_splitzip_encode(n, x, cb, sm, codes, ep, ee);
        CHECK(ne >= 0 && ne <= n);
        or_splitzip_decode(n, cb, sm, codes, ne, ep, ee, y);
        CHECK(n == 0 || memcmp(x, y, (size_t)n * 2) == 0);
        free(x);
        free(y);
        free(sm);
        free(codes);
        free(ep);
        free(ee);
    }

    free(full);
    free(ratio);
    free(kv);
    free(budget);
    free(goh);
    free(chain);
    free(order);
    free(ids);
    free(count);
    free(segp);
    free(goff);
    free(hoff);
    free(table);
    free(kp);
    free(vp);
    free(q);
    free(out);
    free(lse);
    free(lo);
    free(mid);
    free(hi);
    free(po);
    free(pl);
    free(mo);
    free(ml);
    free(sc);
    free(fl);
    free(kq);
    free(vq);
    free(ks);
    free(vs);
    free(k4);
    free(v4);
    free(bytes);
    free(gpu);
}

int main(int argc, char **argv) {
    const int rounds = argc > 1 ? atoi(argv[1]) : 200;
    if (argc > 2) g_state = strtoull(argv[2], NULL, 10);
    for (int r = 0; r < rounds; ++r) round_case();
    printf("oracle fuzz: %d rounds clean\n", rounds);
    return 0;
}
