// Memory-safety drive of the library's host code (allocator, group tables, planner, placement)
// on seeded random inputs, built with AddressSanitizer and UndefinedBehaviorSanitizer by
// tests/test_host_sanitizers.py. Plans are host-only; the device hooks the planner references
// are stubbed below, so no GPU and no CUDA runtime are involved. Any sanitizer report aborts
// with a non-zero status; this program itself checks only what the host API promises (status
// codes, exact page accounting).
// A second drive injects allocation failures: this file replaces the global operator new, and
// while a library call is armed the k-th allocation throws std::bad_alloc, for k = 0, 1, ...
// until the call completes. Every failing call must return TG_ENOMEM, leave the allocator as it
// was and hand back no object, or (where std::stable_sort fell back from a scratch buffer it
// could not get) give the same result as without the failure; the leak check at exit covers
// what a failing call made.
#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <new>
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

// ---- allocation failure injection -------------------------------------------------------
static bool g_armed = false;  // a library call is running under injection
static long g_left = -1;      // allocations left before the injected failure
static bool g_hit = false;    // the injected failure happened
static bool g_hit_nothrow = false;  // ... in a nothrow allocation (the caller may fall back)

static void *counted(std::size_t n, std::size_t align) {
    if (g_armed && g_left >= 0 && g_left-- == 0) {
        g_hit = true;
        throw std::bad_alloc();
    }
    if (n == 0) n = 1;
    void *p = align > alignof(std::max_align_t) ? std::aligned_alloc(align, (n + align - 1) / align * align)
                                                : std::malloc(n);
    if (!p) throw std::bad_alloc();
    return p;
}
static void *counted_nothrow(std::size_t n, std::size_t align) noexcept {
    try {
        return counted(n, align);
    } catch (...) {
        g_hit_nothrow = true;
        return nullptr;
    }
}
void *operator new(std::size_t n) { return counted(n, 0); }
void *operator new[](std::size_t n) { return counted(n, 0); }
void *operator new(std::size_t n, std::align_val_t a) { return counted(n, static_cast<std::size_t>(a)); }
void *operator new[](std::size_t n, std::align_val_t a) { return counted(n, static_cast<std::size_t>(a)); }
void *operator new(std::size_t n, const std::nothrow_t &) noexcept { return counted_nothrow(n, 0); }
void *operator new[](std::size_t n, const std::nothrow_t &) noexcept { return counted_nothrow(n, 0); }
void *operator new(std::size_t n, std::align_val_t a, const std::nothrow_t &) noexcept {
    return counted_nothrow(n, static_cast<std::size_t>(a));
}
void *operator new[](std::size_t n, std::align_val_t a, const std::nothrow_t &) noexcept {
    return counted_nothrow(n, static_cast<std::size_t>(a));
}
void operator delete(void *p) noexcept { std::free(p); }
void operator delete[](void *p) noexcept { std::free(p); }
void operator delete(void *p, std::size_t) noexcept { std::free(p); }
void operator delete[](void *p, std::size_t) noexcept { std::free(p); }
void operator delete(void *p, std::align_val_t) noexcept { std::free(p); }
void operator delete[](void *p, std::align_val_t) noexcept { std::free(p); }
void operator delete(void *p, std::size_t, std::align_val_t) noexcept { std::free(p); }
void operator delete[](void *p, std::size_t, std::align_val_t) noexcept { std::free(p); }
void operator delete(void *p, const std::nothrow_t &) noexcept { std::free(p); }
void operator delete[](void *p, const std::nothrow_t &) noexcept { std::free(p); }

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
    CHECK(tg_alloc_create_ordered(num_pages, 16, order.data(), &a) == TG_OK);
    int32_t seg = -1;
    const int32_t seg_tokens = static_cast<int32_t>(uni(0, 600));
    std::vector<int32_t> seg_pages(static_cast<size_t>(Hkv) * (seg_tokens / 16) + 1);
    CHECK(tg_share_segment(a, seg_tokens, Hkv, &seg, seg_pages.data()) == TG_OK);
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
        std::vector<int32_t> counts(static_cast<size_t>(Hkv), -1);
        const int rc = tg_reserve(a, b, Hkv, kvb.data(), prefixed ? 1 : 0, &seg, out.data(), cap,
                                  counts.data(), &written);
        CHECK(rc == TG_OK || rc == TG_ENOSPC);
        if (rc == TG_ENOSPC) {
            for (int32_t h = 0; h < Hkv; ++h) head_count[static_cast<int64_t>(b) * Hkv + h] = 0;
            continue;
        }
        CHECK(written == cap);
        for (int32_t h = 0; h < Hkv; ++h) {
            CHECK(counts[h] == (kvb[h] + 15) / 16);  // the segment holds whole pages
            head_count[static_cast<int64_t>(b) * Hkv + h] = counts[h];
            kv[static_cast<int64_t>(b) * Hkv + h] = kvb[h];
        }
        ids.insert(ids.end(), out.begin(), out.begin() + cap);
    }
    // reserving a sequence id twice, or more pages than the pool holds, is refused
    std::vector<int32_t> huge(Hkv, static_cast<int32_t>(16 * (num_pages + 1)));
    int64_t w2 = 0;
    std::vector<int32_t> sink(1);
    CHECK(tg_reserve(a, 1000, Hkv, huge.data(), 0, nullptr, sink.data(), 0, nullptr, &w2) != TG_OK);

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
    CHECK(tg_build_group_tables(B, Hkv, head_count.data(), goh.data(), n_groups, ids.data(), table.data(), hoff.data(),
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
    for (int32_t b = 0; b < B; ++b) tg_release(a, b);
    CHECK(tg_release_segment(a, seg) == TG_OK);
    CHECK(tg_alloc_free_pages(a) == num_pages);
    tg_alloc_destroy(a);

    std::vector<int64_t> bytes(B);
    std::vector<int32_t> gpu(B);
    for (auto &x : bytes) x = uni(0, 1 << 20);
    CHECK(tg_place_sequences(B, bytes.data(), static_cast<int32_t>(uni(1, 8)), gpu.data()) == TG_OK);
}

// Runs call() with its k-th allocation failing, for k = 0, 1, ... until a run meets no injected
// failure (its status is returned). After a run that met the failure the status must be
// TG_ENOMEM, or TG_OK where the failure was a nothrow allocation that the call fell back from
// (std::stable_sort's scratch buffer); after(status) then checks the state or the outputs.
template <class Call, class After>
static int under_failures(Call call, After after, long *runs = nullptr) {
    for (long k = 0;; ++k) {
        CHECK(k < 1000000);
        g_left = k;
        g_hit = false;
        g_hit_nothrow = false;
        g_armed = true;
        const int rc = call();
        g_armed = false;
        g_left = -1;
        if (!g_hit) {
            if (runs) *runs += k;
            return rc;
        }
        if (rc != TG_ENOMEM && !(rc == TG_OK && g_hit_nothrow))
            std::fprintf(stderr, "allocation %ld failed: status %d\n", k, rc);
        CHECK(rc == TG_ENOMEM || (rc == TG_OK && g_hit_nothrow));
        after(rc);
    }
}

// A plan's observable content: its counts and its work list.
static std::vector<int64_t> plan_content(const tg_plan *p) {
    tg_plan_info info{};
    CHECK(tg_plan_get_info(p, &info) == TG_OK);
    std::vector<int32_t> items(static_cast<size_t>(info.n_items) * 8 + 1);
    CHECK(tg_plan_items(p, items.data()) == TG_OK);
    std::vector<int64_t> c = {info.n_items, info.n_partials, info.n_merge, info.n_empty, info.n_dynamic,
                              info.n_workers, info.grid, info.n_cascade, info.kv_bytes};
    c.insert(c.end(), items.begin(), items.end());
    return c;
}

static void fault_round(long *runs) {
    const int32_t B = static_cast<int32_t>(uni(1, 4)), Hkv = static_cast<int32_t>(uni(1, 4));
    const int64_t BH = static_cast<int64_t>(B) * Hkv;
    const int64_t num_pages = 300 + uni(0, 100);
    tg_alloc *a = nullptr;
    // the seeded form (it shuffles in a temporary order vector first), then the ordered form
    CHECK(under_failures([&] { return tg_alloc_create(num_pages, 16, static_cast<uint64_t>(num_pages), &a); },
                         [&](int) { CHECK(!a); }, runs) == TG_OK);
    tg_alloc_destroy(a);
    a = nullptr;
    CHECK(under_failures([&] { return tg_alloc_create_ordered(num_pages, 16, nullptr, &a); }, [&](int) { CHECK(!a); }, runs) ==
          TG_OK);
    auto refs = [&] {
        std::vector<int32_t> r(static_cast<size_t>(num_pages));
        for (int64_t i = 0; i < num_pages; ++i) r[i] = tg_alloc_refcount(a, static_cast<int32_t>(i));
        return r;
    };
    auto consistent = [&] {
        int64_t held = 0;
        for (int64_t i = 0; i < num_pages; ++i) held += tg_alloc_refcount(a, static_cast<int32_t>(i)) > 0;
        CHECK(held + tg_alloc_free_pages(a) == num_pages);
    };
    // a shared segment, then every sequence (half of them on the segment)
    std::vector<int32_t> before = refs();
    int64_t free_before = tg_alloc_free_pages(a);
    const int32_t seg_tokens = 64 + static_cast<int32_t>(uni(0, 15));
    int32_t seg = -1;
    std::vector<int32_t> seg_pages(static_cast<size_t>(Hkv) * 4);
    CHECK(under_failures([&] { return tg_share_segment(a, seg_tokens, Hkv, &seg, seg_pages.data()); },
                         [&](int) { CHECK(refs() == before && tg_alloc_free_pages(a) == free_before); }, runs) ==
          TG_OK);
    consistent();
    std::vector<int32_t> kv(static_cast<size_t>(BH)), ids, head_count(static_cast<size_t>(BH));
    for (int32_t b = 0; b < B; ++b) {
        std::vector<int32_t> kvb(static_cast<size_t>(Hkv));
        for (auto &x : kvb) x = 64 + static_cast<int32_t>(uni(0, 300));
        const int32_t segs[1] = {b % 2 ? seg : -1};
        int64_t cap = 0;
        for (int32_t x : kvb) cap += (x + 15) / 16;
        std::vector<int32_t> out(static_cast<size_t>(cap));
        int64_t written = 0;
        before = refs();
        free_before = tg_alloc_free_pages(a);
        CHECK(under_failures(
                  [&] { return tg_reserve(a, b, Hkv, kvb.data(), 1, segs, out.data(), cap, nullptr, &written); },
                  [&](int) {
                      CHECK(refs() == before && tg_alloc_free_pages(a) == free_before);
                      CHECK(tg_release(a, b) == TG_ENOTFOUND);
                  },
                  runs) == TG_OK);
        CHECK(written == cap);
        consistent();
        for (int32_t h = 0; h < Hkv; ++h) {
            kv[static_cast<int64_t>(b) * Hkv + h] = kvb[h];
            head_count[static_cast<int64_t>(b) * Hkv + h] = (kvb[h] + 15) / 16;
        }
        ids.insert(ids.end(), out.begin(), out.end());
    }
    // budget groups, group tables, placement (outputs only)
    const int32_t n_groups = static_cast<int32_t>(uni(1, Hkv));
    std::vector<int32_t> budget(static_cast<size_t>(Hkv)), goh(static_cast<size_t>(Hkv));
    for (auto &x : budget) x = static_cast<int32_t>(uni(0, 1000000));
    CHECK(tg_budget_groups(Hkv, budget.data(), n_groups, goh.data()) == TG_OK);
    const std::vector<int32_t> goh_expect = goh;
    CHECK(under_failures([&] { return tg_budget_groups(Hkv, budget.data(), n_groups, goh.data()); },
                         [&](int rc) { CHECK(rc != TG_OK || goh == goh_expect); }, runs) == TG_OK);
    CHECK(goh == goh_expect);
    std::vector<int64_t> goff(static_cast<size_t>(n_groups) + 1), hoff(static_cast<size_t>(BH));
    CHECK(tg_build_group_tables(B, Hkv, head_count.data(), goh.data(), n_groups, ids.data(), nullptr, hoff.data(),
                          goff.data()) == TG_OK);
    const int64_t tsize = goff[n_groups];
    std::vector<int32_t> table(static_cast<size_t>(tsize) + 1);
    CHECK(under_failures([&] {
              return tg_build_group_tables(B, Hkv, head_count.data(), goh.data(), n_groups, ids.data(), table.data(),
                                     hoff.data(), goff.data());
          },
          [](int rc) { CHECK(rc == TG_ENOMEM); }, runs) == TG_OK);
    std::vector<int64_t> bytes(static_cast<size_t>(B));
    std::vector<int32_t> gpu(static_cast<size_t>(B));
    for (auto &x : bytes) x = uni(0, 1 << 20);
    CHECK(tg_place_sequences(B, bytes.data(), 2, gpu.data()) == TG_OK);
    const std::vector<int32_t> gpu_expect = gpu;
    CHECK(under_failures([&] { return tg_place_sequences(B, bytes.data(), 2, gpu.data()); },
                         [&](int rc) { CHECK(rc != TG_OK || gpu == gpu_expect); }, runs) == TG_OK);
    CHECK(gpu == gpu_expect);

    // plans: bf16 split, whole heads, tiered INT8 / INT4, cascade; a failing call hands back none
    tg_shape s{};
    s.B = B;
    s.Hkv = Hkv;
    s.Hq = Hkv * 4;
    s.D = 128;
    s.page = 16;
    s.num_pages = num_pages;
    std::vector<int32_t> fl(static_cast<size_t>(BH));
    for (auto &x : fl) x = static_cast<int32_t>(uni(0, 100));
    for (int variant = 0; variant < 5; ++variant) {
        tg_plan_opts o{};
        o.host_only = 1;
        o.num_workers = static_cast<int32_t>(uni(1, 300));
        o.min_splits = static_cast<int32_t>(uni(1, 4));
        o.whole_heads = variant == 1;
        o.slow_bits = variant == 3 ? 4 : 0;
        tg_shape st = s;
        if (variant == 2 || variant == 3) st.num_slow_pages = num_pages;
        tg_plan *p = nullptr;
        auto create = [&] {
            if (variant == 4)
                return tg_plan_create_cascade(&st, kv.data(), goh.data(), goff.data(), n_groups, table.data(),
                                              hoff.data(), tsize, 2, &o, &p);
            return tg_plan_create(&st, kv.data(), variant == 2 || variant == 3 ? fl.data() : nullptr, goh.data(),
                                  goff.data(), n_groups, variant >= 2 ? tsize + 1 : 0, &o, &p);
        };
        CHECK(create() == TG_OK && p);
        const std::vector<int64_t> expect = plan_content(p);
        tg_plan_destroy(p);
        p = nullptr;
        const int rc = under_failures(create,
                                      [&](int r) {
                                          if (r == TG_OK) {  // a sort fell back: the same plan
                                              CHECK(p && plan_content(p) == expect);
                                              tg_plan_destroy(p);
                                              p = nullptr;
                                          } else {
                                              CHECK(!p);
                                          }
                                      },
                                      runs);
        CHECK(rc == TG_OK && p && plan_content(p) == expect);
        tg_plan_destroy(p);
    }

    for (int32_t b = 0; b < B; ++b) CHECK(tg_release(a, b) == TG_OK);
    CHECK(tg_release_segment(a, seg) == TG_OK);
    CHECK(tg_alloc_free_pages(a) == num_pages);
    tg_alloc_destroy(a);
}

int main(int argc, char **argv) {
    const int rounds = argc > 1 ? std::atoi(argv[1]) : 300;
    if (argc > 2) rng.seed(std::strtoull(argv[2], nullptr, 10));
    for (int r = 0; r < rounds; ++r) admission_round();
    std::printf("host fuzz: %d rounds clean\n", rounds);
    const int fault_rounds = argc > 3 ? std::atoi(argv[3]) : 20;
    long runs = 0;
    for (int r = 0; r < fault_rounds; ++r) fault_round(&runs);
    std::printf("allocation failures: %d rounds, %ld injected, each TG_ENOMEM with state kept or absorbed\n",
                fault_rounds, runs);
    return 0;
}
