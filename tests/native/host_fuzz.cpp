// Memory-safety drive of the library's host code (allocator, group tables, planner, placement)
// on seeded random inputs, built with AddressSanitizer and UndefinedBehaviorSanitizer by
// tests/test_host_sanitizers.py. Plans are host-only; the device hooks the planner references
// are stubbed below, so no GPU and no CUDA runtime are involved. Any sanitizer report aborts
// with a non-zero status; the driver itself checks only what the host API promises (status
// codes, exact page accounting).
#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <random>
#include <vector>

#include "tg.h"
#include "tg_internal.h"

namespace tg {
int device_init_plan(tg_plan *) { return TG_EUNSUPPORTED; }
void device_free_plan(tg_plan *) {}
int device_num_sms(int, int *num_sms) {
    *num_sms = 148;
    return TG_OK;
}
void set_cuda_error(const char *, int) {}
}  // namespace tg

#define CHECK(c)                                                                      \
    do {                                                                              \
        if (!(c)) {                                                                   \
            std::fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c);     \
            std::exit(2);                                                             \
        }                                                                             \
    } while (0)

static std::mt19937_64 rng(20261202);
static int64_t uni(int64_t lo, int64_t hi) { return std::uniform_int_distribution<int64_t>(lo, hi)(rng); }

static void admission_round() {
    const int32_t B = static_cast<int32_t>(uni(1, 6)), Hkv = static_cast<int32_t>(uni(1, 8));
    const int64_t BH = static_cast<int64_t>(B) * Hkv;
    std::vector<int32_t> full(BH), ratio(BH), kv(BH);
    for (int64_t i = 0; i < BH; ++i) {
        full[i] = static_cast<int32_t>(uni(0, 900));
        ratio[i] = static_cast<int32_t>(uni(0, 1000000));
    }
    CHECK(tg_retained_lengths(BH, full.data(), ratio.data(), kv.data()) == TG_OK);
    for (int64_t i = 0; i < BH; ++i) CHECK(kv[i] >= 0 && kv[i] <= full[i]);
    const int32_t n_groups = static_cast<int32_t>(uni(1, Hkv));
    std::vector<int32_t> budget(Hkv), goh(Hkv);
    for (auto &b : budget) b = static_cast<int32_t>(uni(0, 1000000));
    CHECK(tg_budget_groups(Hkv, budget.data(), n_groups, goh.data()) == TG_OK);

    // allocator: an optional shared segment, then every sequence, some released again
    int64_t need = 0;
    for (int64_t i = 0; i < BH; ++i) need += (kv[i] + 15) / 16;
    const int64_t num_pages = need + uni(0, 64) + 40 * Hkv;
    std::vector<int32_t> order(num_pages);
    for (int64_t i = 0; i < num_pages; ++i) order[i] = static_cast<int32_t>(i);
    std::shuffle(order.begin(), order.end(), rng);
    tg_alloc *a = nullptr;
    CHECK(tg_alloc_create(num_pages, 16, order.data(), &a) == TG_OK);
    int32_t seg = -1;
    const int32_t seg_tokens = static_cast<int32_t>(uni(0, 600));
    std::vector<int32_t> seg_pages(static_cast<size_t>(Hkv) * (seg_tokens / 16) + 1);
    CHECK(tg_alloc_share_segment(a, seg_tokens, Hkv, &seg, seg_pages.data()) == TG_OK);
    std::vector<int32_t> ids;
    std::vector<int32_t> head_count(BH);
    for (int32_t b = 0; b < B; ++b) {
        const bool prefixed = uni(0, 1) == 1;
        std::vector<int32_t> kvb(kv.begin() + static_cast<int64_t>(b) * Hkv, kv.begin() + static_cast<int64_t>(b + 1) * Hkv);
        if (prefixed)
            for (auto &x : kvb) x = std::max(x, seg_tokens);
        int64_t cap = 0;
        for (int32_t x : kvb) cap += (x + 15) / 16;
        std::vector<int32_t> out(static_cast<size_t>(cap) + 1);
        int64_t written = -1;
        const int rc = tg_alloc_reserve(a, b, Hkv, kvb.data(), prefixed ? 1 : 0, &seg, out.data(), cap, &written);
        CHECK(rc == TG_OK || rc == TG_ENOSPC);
        if (rc == TG_ENOSPC) {
            for (int32_t h = 0; h < Hkv; ++h) head_count[static_cast<int64_t>(b) * Hkv + h] = 0;
            continue;
        }
        CHECK(written == cap);
        for (int32_t h = 0; h < Hkv; ++h) {
            head_count[static_cast<int64_t>(b) * Hkv + h] = (kvb[h] + 15) / 16;
            kv[static_cast<int64_t>(b) * Hkv + h] = kvb[h];
        }
        ids.insert(ids.end(), out.begin(), out.begin() + cap);
    }
    // reserving a sequence id twice, or more pages than the pool holds, is refused
    std::vector<int32_t> huge(Hkv, static_cast<int32_t>(16 * (num_pages + 1)));
    int64_t w2 = 0;
    std::vector<int32_t> sink(1);
    CHECK(tg_alloc_reserve(a, 1000, Hkv, huge.data(), 0, nullptr, sink.data(), 0, &w2) != TG_OK);

    // group tables over what was reserved
    std::vector<int64_t> goff(static_cast<size_t>(n_groups) + 1);
    int64_t tsize = 0;
    for (int32_t g = 0; g < n_groups; ++g) {
        int64_t hg = 0, pg = 0;
        for (int32_t h = 0; h < Hkv; ++h)
            if (goh[h] == g) {
                ++hg;
                for (int32_t b = 0; b < B; ++b) pg = std::max<int64_t>(pg, head_count[static_cast<int64_t>(b) * Hkv + h]);
            }
        tsize += static_cast<int64_t>(B) * hg * pg;
    }
    std::vector<int32_t> table(static_cast<size_t>(tsize) + 1);
    std::vector<int64_t> hoff(BH);
    CHECK(tg_group_tables(B, Hkv, head_count.data(), goh.data(), n_groups, ids.data(), table.data(), hoff.data(),
                          goff.data()) == TG_OK);

    // plans: bf16 (static, hybrid, whole heads), tiered INT8 / INT4, cascade
    const int32_t G = 1 << uni(0, 3);   // the kernels serve 1, 2, 4 or 8 query heads per KV head
    tg_shape s{};
    s.B = B;
    s.Hq = Hkv * G;
    s.Hkv = Hkv;
    s.D = uni(0, 1) ? 128 : 64;
    s.page = 16;
    s.num_pages = num_pages;
    for (int32_t h = 0; h < B * Hkv; ++h)
        if (head_count[h] == 0) kv[h] = 0;
    for (int trial = 0; trial < 4; ++trial) {
        tg_plan_opts o{};
        o.host_only = 1;
        o.num_workers = static_cast<int32_t>(uni(1, 400));
        o.min_splits = static_cast<int32_t>(uni(1, 9));
        o.max_chunk_pages = static_cast<int32_t>(uni(0, 20));
        o.static_permille = static_cast<int32_t>(uni(0, 1000));
        o.dyn_chunk_pages = static_cast<int32_t>(uni(0, 16));
        o.whole_heads = trial == 3;
        tg_plan *p = nullptr;
        const int rc = tg_plan_create(&s, kv.data(), nullptr, goh.data(), goff.data(), n_groups, 0, &o, &p);
        CHECK(rc == TG_OK);
        tg_plan_info info{};
        CHECK(tg_plan_get_info(p, &info) == TG_OK);
        std::vector<int32_t> items(static_cast<size_t>(info.n_items) * 8 + 8);
        CHECK(tg_plan_items(p, items.data()) == TG_OK);
        tg_plan_destroy(p);
    }
    {   // unsupported shapes are refused, and no plan comes back
        tg_shape bad = s;
        bad.Hq = Hkv * 3;
        int sentinel = 0;
        tg_plan *p = reinterpret_cast<tg_plan *>(&sentinel);
        CHECK(tg_plan_create(&bad, kv.data(), nullptr, goh.data(), goff.data(), n_groups, 0, nullptr, &p) ==
              TG_EUNSUPPORTED);
        CHECK(p == nullptr);
        bad = s;
        bad.D = 96;
        p = reinterpret_cast<tg_plan *>(&sentinel);
        CHECK(tg_plan_create(&bad, kv.data(), nullptr, goh.data(), goff.data(), n_groups, 0, nullptr, &p) ==
              TG_EUNSUPPORTED);
        CHECK(p == nullptr);
    }
    {
        tg_shape st = s;
        st.D = 128;
        std::vector<int32_t> fl(BH);
        for (int64_t i = 0; i < BH; ++i) fl[i] = static_cast<int32_t>(uni(0, 300));
        st.num_slow_pages = num_pages;
        for (int bits : {8, 4}) {
            tg_plan_opts o{};
            o.host_only = 1;
            o.num_workers = static_cast<int32_t>(uni(1, 400));
            o.min_splits = static_cast<int32_t>(uni(1, 9));
            o.slow_bits = bits;
            o.capacity = static_cast<int32_t>(uni(0, 1));
            tg_plan *p = nullptr;
            CHECK(tg_plan_create(&st, kv.data(), fl.data(), goh.data(), goff.data(), n_groups, tsize + 1, &o, &p) == TG_OK);
            tg_plan_destroy(p);
        }
    }
    if (tsize > 0) {
        tg_plan_opts o{};
        o.host_only = 1;
        o.num_workers = static_cast<int32_t>(uni(1, 400));
        tg_plan *p = nullptr;
        const int rc = tg_plan_create_cascade(&s, kv.data(), goh.data(), goff.data(), n_groups, table.data(), hoff.data(),
                                              tsize, 2, &o, &p);
        CHECK(rc == TG_OK);
        tg_plan_info info{};
        CHECK(tg_plan_get_info(p, &info) == TG_OK);
        std::vector<int32_t> units(static_cast<size_t>(info.n_cascade) * (4 + 2 * 256) + 1);
        CHECK(tg_plan_cascade_units(p, units.data()) == TG_OK);
        tg_plan_destroy(p);
    }

    // release everything; every page returns to the free list
    for (int32_t b = 0; b < B; ++b) tg_alloc_release(a, b);
    CHECK(tg_alloc_release_segment(a, seg) == TG_OK);
    CHECK(tg_alloc_free_pages(a) == num_pages);
    tg_alloc_destroy(a);

    std::vector<int64_t> bytes(B);
    std::vector<int32_t> gpu(B);
    for (auto &x : bytes) x = uni(0, 1 << 20);
    CHECK(tg_place_sequences(B, bytes.data(), static_cast<int32_t>(uni(1, 8)), gpu.data()) == TG_OK);
}

int main(int argc, char **argv) {
    const int rounds = argc > 1 ? std::atoi(argv[1]) : 300;
    if (argc > 2) rng.seed(std::strtoull(argv[2], nullptr, 10));
    for (int r = 0; r < rounds; ++r) admission_round();
    std::printf("host fuzz: %d rounds clean\n", rounds);
    return 0;
}
