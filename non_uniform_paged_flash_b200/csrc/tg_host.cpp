// Host side of libtg: admission-time steps (retained lengths, budget groups, the
// budget-reservation allocator, group page tables, AOT placement) and the static work-list
// planner. Pure host C++; the CUDA side lives in tg_kernels.cu.
#include <algorithm>
#include <climits>
#include <cstring>
#include <memory>
#include <new>
#include <numeric>
#include <unordered_map>
#include <vector>

#include "tg_internal.h"

// ------------------------------------------------------------------------------------------
// Status text
// ------------------------------------------------------------------------------------------
extern "C" const char *tg_strerror(int s) {
    switch (s) {
        case TG_OK: return "ok";
        case TG_EINVAL: return "invalid argument";
        case TG_ENOSPC: return "page pool exhausted";
        case TG_EBADPAGE: return "page id, table row or length outside the plan (pages skipped)";
        case TG_ECUDA: return "CUDA runtime error";
        case TG_ETIMEOUT: return "kernel wait timed out";
        case TG_ENOMEM: return "out of memory";
        case TG_ENOTFOUND: return "unknown sequence or segment";
        case TG_EUNSUPPORTED: return "unsupported shape";
        case TG_EEXIST: return "sequence already reserved";
        default: return "unknown status";
    }
}

// ------------------------------------------------------------------------------------------
// Retained length from the budget table ("Tangram": per-head ratio fixed at admission).
// ------------------------------------------------------------------------------------------
extern "C" int tg_retained_lengths(int64_t n, const int32_t *full_len, const int32_t *ratio_ppm,
                                   int32_t *kv_len) {
    if (n < 0 || (n > 0 && (!full_len || !ratio_ppm || !kv_len))) return TG_EINVAL;
    for (int64_t i = 0; i < n; ++i)
        if (ratio_ppm[i] < 0 || ratio_ppm[i] > 1000000) return TG_EINVAL;
    for (int64_t i = 0; i < n; ++i) {
        const int64_t L = full_len[i];
        if (L <= 0) { kv_len[i] = 0; continue; }
        int64_t r = (static_cast<int64_t>(ratio_ppm[i]) * L + 500000) / 1000000;
        kv_len[i] = static_cast<int32_t>(std::min<int64_t>(L, std::max<int64_t>(1, r)));
    }
    return TG_OK;
}

// ------------------------------------------------------------------------------------------
// Budget groups (Ragged Paging): equal-count quantiles of the budget ranking.
// ------------------------------------------------------------------------------------------
extern "C" int tg_budget_groups(int32_t n, const int32_t *budget_ppm, int32_t n_groups,
                                int32_t *group_of_head) {
    return tg::no_throw([&] {
        if (n <= 0 || !budget_ppm || !group_of_head || n_groups < 1 || n_groups > n) return TG_EINVAL;
        std::vector<int32_t> order(n);
        std::iota(order.begin(), order.end(), 0);
        std::stable_sort(order.begin(), order.end(),
                         [&](int32_t a, int32_t b) { return budget_ppm[a] < budget_ppm[b]; });
        for (int32_t pos = 0; pos < n; ++pos)
            group_of_head[order[pos]] = static_cast<int32_t>(static_cast<int64_t>(pos) * n_groups / n);
        return TG_OK;
    });
}

// ------------------------------------------------------------------------------------------
// Budget-reservation allocator.
// ------------------------------------------------------------------------------------------
struct tg_alloc {
    int64_t num_pages = 0;
    int32_t page = 16;
    // Free pages in FIFO order: a ring of num_pages entries (a page is in it at most once), so
    // that returning a page never allocates.
    std::vector<int32_t> ring;
    int64_t head = 0, n_free = 0;
    std::vector<int32_t> refs;
    struct Segment {
        int32_t n_heads = 0, full = 0;
        bool alive = false;
        std::vector<int32_t> pages;  // [n_heads][full]
    };
    std::vector<Segment> segs;
    struct Seq {
        std::vector<int32_t> priv;    // private pages in allocation order
        std::vector<int32_t> shared;  // shared page references held
    };
    std::unordered_map<int32_t, Seq> seqs;

    int32_t take() {
        const int32_t p = ring[head];
        head = head + 1 == num_pages ? 0 : head + 1;
        --n_free;
        return p;
    }
    void give(int32_t p) {
        int64_t at = head + n_free;
        if (at >= num_pages) at -= num_pages;
        ring[at] = p;
        ++n_free;
    }
    void unref(int32_t p) {
        if (--refs[p] == 0) give(p);
    }
};

namespace {

int alloc_create(int64_t num_pages, int32_t page, const int32_t *free_order, tg_alloc **out) {
    if (!out || num_pages < 1 || num_pages > INT32_MAX || page < 1) return TG_EINVAL;
    std::unique_ptr<tg_alloc> a(new tg_alloc);
    a->num_pages = num_pages;
    a->page = page;
    a->refs.assign(static_cast<size_t>(num_pages), 0);
    a->ring.assign(static_cast<size_t>(num_pages), 0);
    std::vector<char> seen(static_cast<size_t>(num_pages), 0);
    for (int64_t i = 0; i < num_pages; ++i) {
        const int32_t p = free_order ? free_order[i] : static_cast<int32_t>(i);
        if (p < 0 || p >= num_pages || seen[p]) return TG_EINVAL;
        seen[p] = 1;
        a->give(p);
    }
    *out = a.release();
    return TG_OK;
}

int alloc_share_segment(tg_alloc *a, int32_t n_tokens, int32_t n_heads, int32_t *seg_id,
                        int32_t *page_ids) {
    if (!a || !seg_id || n_tokens < 0 || n_heads < 1) return TG_EINVAL;
    const int32_t full = n_tokens / a->page;
    const int64_t need = static_cast<int64_t>(full) * n_heads;
    if (need > a->n_free) return TG_ENOSPC;
    std::vector<int32_t> pages;
    pages.reserve(static_cast<size_t>(need));  // the fallible steps come first
    a->segs.emplace_back();
    tg_alloc::Segment &s = a->segs.back();
    s.n_heads = n_heads;
    s.full = full;
    s.alive = true;
    for (int64_t i = 0; i < need; ++i) {
        const int32_t p = a->take();
        a->refs[p] = 1;  // the segment's own reference
        pages.push_back(p);
    }
    if (page_ids && need > 0) std::memcpy(page_ids, pages.data(), sizeof(int32_t) * static_cast<size_t>(need));
    s.pages = std::move(pages);
    *seg_id = static_cast<int32_t>(a->segs.size() - 1);
    return TG_OK;
}

int alloc_reserve(tg_alloc *a, int32_t seq_id, int32_t n_heads, const int32_t *kv_len, int32_t n_prefix,
                  const int32_t *prefix_segs, int32_t *page_ids, int64_t capacity, int32_t *head_count,
                  int64_t *n_written) {
    if (!a || n_heads < 1 || !kv_len || n_prefix < 0 || (n_prefix > 0 && !prefix_segs) ||
        (capacity > 0 && !page_ids) || capacity < 0)
        return TG_EINVAL;
    if (a->seqs.count(seq_id)) return TG_EEXIST;
    int64_t shared_pages = 0;
    for (int32_t c = 0; c < n_prefix; ++c) {
        const int32_t s = prefix_segs[c];
        if (s < 0) continue;
        if (s >= static_cast<int32_t>(a->segs.size()) || !a->segs[s].alive) return TG_ENOTFOUND;
        if (a->segs[s].n_heads != n_heads) return TG_EINVAL;
        shared_pages += a->segs[s].full;
    }
    const int64_t shared_tokens = shared_pages * a->page;
    int64_t priv_total = 0, total = 0;
    for (int32_t h = 0; h < n_heads; ++h) {
        if (kv_len[h] < shared_tokens) return TG_EINVAL;
        const int64_t priv = (kv_len[h] - shared_tokens + a->page - 1) / a->page;
        priv_total += priv;
        total += shared_pages + priv;
    }
    if (total > capacity) return TG_EINVAL;
    if (priv_total > a->n_free) return TG_ENOSPC;

    // The fallible steps (the sequence's record and its page lists) before any page moves.
    tg_alloc::Seq &sq = a->seqs[seq_id];
    try {
        sq.shared.reserve(static_cast<size_t>(shared_pages) * static_cast<size_t>(n_heads));
        sq.priv.reserve(static_cast<size_t>(priv_total));
    } catch (...) {
        a->seqs.erase(seq_id);
        throw;
    }
    int64_t w = 0;
    for (int32_t h = 0; h < n_heads; ++h) {
        for (int32_t c = 0; c < n_prefix; ++c) {
            const int32_t s = prefix_segs[c];
            if (s < 0) continue;
            const tg_alloc::Segment &sg = a->segs[s];
            for (int32_t p = 0; p < sg.full; ++p) {
                const int32_t id = sg.pages[static_cast<size_t>(h) * sg.full + p];
                ++a->refs[id];
                sq.shared.push_back(id);
                page_ids[w++] = id;
            }
        }
        const int64_t priv = (kv_len[h] - shared_tokens + a->page - 1) / a->page;
        for (int64_t p = 0; p < priv; ++p) {
            const int32_t id = a->take();
            a->refs[id] = 1;
            sq.priv.push_back(id);
            page_ids[w++] = id;
        }
        if (head_count) head_count[h] = static_cast<int32_t>(shared_pages + priv);
    }
    if (n_written) *n_written = w;
    return TG_OK;
}

}  // namespace

extern "C" int tg_alloc_create_ordered(int64_t num_pages, int32_t page, const int32_t *free_order,
                                       tg_alloc **out) {
    return tg::no_throw([&] { return alloc_create(num_pages, page, free_order, out); });
}

// SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number generators", 2014):
// the state advances by the golden-ratio increment and each output is the state's 64-bit
// finaliser (two xor-shift-multiply rounds and a final xor-shift).
static uint64_t splitmix64_next(uint64_t &state) {
    uint64_t z = (state += 0x9E3779B97F4A7C15ULL);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

extern "C" int tg_alloc_create(int64_t num_pages, int32_t page, uint64_t seed, tg_alloc **out) {
    return tg::no_throw([&] {
        if (!out || num_pages < 1 || num_pages > INT32_MAX || page < 1) return TG_EINVAL;
        // Durstenfeld's in-place Fisher-Yates shuffle, the k-th swap drawing the k-th output.
        std::vector<int32_t> order(static_cast<size_t>(num_pages));
        for (int64_t i = 0; i < num_pages; ++i) order[static_cast<size_t>(i)] = static_cast<int32_t>(i);
        uint64_t state = seed;
        for (int64_t i = num_pages - 1; i >= 1; --i) {
            const int64_t j = static_cast<int64_t>(splitmix64_next(state) % static_cast<uint64_t>(i + 1));
            std::swap(order[static_cast<size_t>(i)], order[static_cast<size_t>(j)]);
        }
        return alloc_create(num_pages, page, order.data(), out);
    });
}

extern "C" void tg_alloc_destroy(tg_alloc *a) { delete a; }

extern "C" int64_t tg_alloc_free_pages(const tg_alloc *a) { return a ? a->n_free : -1; }

extern "C" int32_t tg_alloc_refcount(const tg_alloc *a, int32_t page_id) {
    if (!a || page_id < 0 || page_id >= a->num_pages) return -1;
    return a->refs[page_id];
}

extern "C" int tg_share_segment(tg_alloc *a, int32_t n_tokens, int32_t n_heads, int32_t *seg_id,
                                int32_t *page_ids) {
    return tg::no_throw([&] { return alloc_share_segment(a, n_tokens, n_heads, seg_id, page_ids); });
}

extern "C" int tg_reserve(tg_alloc *a, int32_t seq_id, int32_t n_heads, const int32_t *kv_len,
                          int32_t n_prefix, const int32_t *prefix_segs, int32_t *page_ids,
                          int64_t capacity, int32_t *head_count, int64_t *n_written) {
    return tg::no_throw([&] {
        return alloc_reserve(a, seq_id, n_heads, kv_len, n_prefix, prefix_segs, page_ids, capacity,
                             head_count, n_written);
    });
}

extern "C" int tg_release(tg_alloc *a, int32_t seq_id) {
    if (!a) return TG_EINVAL;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return TG_ENOTFOUND;
    for (int32_t p : it->second.priv) a->unref(p);
    for (int32_t p : it->second.shared) a->unref(p);
    a->seqs.erase(it);
    return TG_OK;
}

extern "C" int tg_release_segment(tg_alloc *a, int32_t seg_id) {
    if (!a) return TG_EINVAL;
    if (seg_id < 0 || seg_id >= static_cast<int32_t>(a->segs.size()) || !a->segs[seg_id].alive)
        return TG_ENOTFOUND;
    tg_alloc::Segment &s = a->segs[seg_id];
    s.alive = false;
    for (int32_t p : s.pages) a->unref(p);
    return TG_OK;
}

// ------------------------------------------------------------------------------------------
// Group page tables (Ragged Paging).
// ------------------------------------------------------------------------------------------
extern "C" int tg_build_group_tables(int32_t B, int32_t Hkv, const int32_t *head_count,
                                     const int32_t *group_of_head, int32_t n_groups,
                                     const int32_t *page_ids, int32_t *table, int64_t *head_off,
                                     int64_t *group_off) {
    return tg::no_throw([&] {
        if (B < 0 || Hkv < 1 || !head_count || !group_of_head || n_groups < 1 || !group_off)
            return TG_EINVAL;
        for (int32_t h = 0; h < Hkv; ++h)
            if (group_of_head[h] < 0 || group_of_head[h] >= n_groups) return TG_EINVAL;
        const int64_t BH = static_cast<int64_t>(B) * Hkv;
        std::vector<int64_t> src(static_cast<size_t>(BH) + 1, 0);
        for (int64_t i = 0; i < BH; ++i) {
            if (head_count[i] < 0) return TG_EINVAL;
            src[i + 1] = src[i] + head_count[i];
        }
        if (table && (!page_ids || !head_off)) return TG_EINVAL;
        int64_t pos = 0;
        for (int32_t g = 0; g < n_groups; ++g) {
            group_off[g] = pos;
            std::vector<int32_t> heads;
            int64_t Pg = 0;
            for (int32_t h = 0; h < Hkv; ++h) {
                if (group_of_head[h] != g) continue;
                heads.push_back(h);
                for (int32_t b = 0; b < B; ++b)
                    Pg = std::max<int64_t>(Pg, head_count[static_cast<int64_t>(b) * Hkv + h]);
            }
            const int64_t Hg = static_cast<int64_t>(heads.size());
            if (table) {
                for (int32_t b = 0; b < B; ++b)
                    for (int64_t j = 0; j < Hg; ++j) {
                        const int64_t bh = static_cast<int64_t>(b) * Hkv + heads[j];
                        const int64_t row = pos + (static_cast<int64_t>(b) * Hg + j) * Pg;
                        head_off[bh] = row;
                        const int64_t cnt = head_count[bh];
                        for (int64_t p = 0; p < Pg; ++p)
                            table[row + p] = p < cnt ? page_ids[src[bh] + p] : -1;
                    }
            } else if (head_off) {
                for (int32_t b = 0; b < B; ++b)
                    for (int64_t j = 0; j < Hg; ++j)
                        head_off[static_cast<int64_t>(b) * Hkv + heads[j]] =
                            pos + (static_cast<int64_t>(b) * Hg + j) * Pg;
            }
            pos += static_cast<int64_t>(B) * Hg * Pg;
        }
        group_off[n_groups] = pos;
        return TG_OK;
    });
}

// ------------------------------------------------------------------------------------------
// AOT placement of sequences on GPUs (LPT greedy).
// ------------------------------------------------------------------------------------------
extern "C" int tg_place_sequences(int32_t n_seq, const int64_t *seq_bytes, int32_t n_gpus,
                                  int32_t *gpu_of_seq) {
    return tg::no_throw([&] {
        if (n_seq < 0 || n_gpus < 1 || (n_seq > 0 && (!seq_bytes || !gpu_of_seq))) return TG_EINVAL;
        std::vector<int32_t> order(n_seq);
        std::iota(order.begin(), order.end(), 0);
        std::stable_sort(order.begin(), order.end(),
                         [&](int32_t a, int32_t b) { return seq_bytes[a] > seq_bytes[b]; });
        std::vector<int64_t> load(n_gpus, 0);
        for (int32_t s : order) {
            const int32_t g = static_cast<int32_t>(std::min_element(load.begin(), load.end()) - load.begin());
            gpu_of_seq[s] = g;
            load[g] += seq_bytes[s];
        }
        return TG_OK;
    });
}

// ------------------------------------------------------------------------------------------
// Static work-list planner.
//
// Each head's tokens are cut into chunks (per tier; chunks never cross the tier boundary),
// then the byte cost of the chunks, in (sequence, head, tier, chunk) order, is cut into
// num_workers contiguous ranges of equal cost. A chunk that straddles a range boundary is
// cut at the page nearest the boundary. Every resulting (worker, chunk piece) is an item.
// ------------------------------------------------------------------------------------------
namespace tg {

// Partial slots and the merge list: a head's items are consecutive in the list.
// A cascade head's partials come first (slots first_slot .. first_slot + casc_cnt - 1, in
// the order of its cascade runs), then its items'.
static int finish_slots(tg_plan *p, const int32_t *casc_cnt) {
    const int64_t BH = static_cast<int64_t>(p->shape.B) * p->shape.Hkv;
    std::vector<int32_t> cnt(static_cast<size_t>(BH), 0), first(static_cast<size_t>(BH), -1);
    for (size_t i = 0; i < p->items.size(); ++i) {
        const int32_t bh = p->items[i].bh;
        if (first[bh] < 0) first[bh] = static_cast<int32_t>(i);
        ++cnt[bh];
    }
    p->merge.clear();
    p->empties.clear();
    p->merge_warps = 1;
    int64_t slot = 0;
    for (int64_t bh = 0; bh < BH; ++bh) {
        const int32_t cc = casc_cnt ? casc_cnt[bh] : 0;
        const int32_t total = cnt[bh] + cc;
        if (total == 0) {
            p->empties.push_back(static_cast<int32_t>(bh));
        } else if (total > 1 || cc > 0) {
            const int32_t mi = static_cast<int32_t>(p->merge.size());
            p->merge.push_back({static_cast<int32_t>(bh), static_cast<int32_t>(slot), total, 0});
            slot += cc;
            for (int32_t j = 0; j < cnt[bh]; ++j) {
                Item &it = p->items[first[bh] + j];
                it.slot = static_cast<int32_t>(slot++);
                it.flags |= mi << 1;
            }
            // warps per merge CTA: up to 8 splits per warp, at most 32 warps
            p->merge_warps = std::max(p->merge_warps, std::min(32, (total + 7) / 8));
        }
    }
    p->n_partials = slot;
    return TG_OK;
}

int build_work_list(tg_plan *p, const int32_t *kv_len, const int32_t *fast_len,
                    int32_t num_workers, int32_t min_splits, int32_t max_chunk_pages,
                    int32_t static_permille, int32_t dyn_chunk_pages, const int32_t *pstart,
                    const int32_t *casc_cnt) {
    const tg_shape &s = p->shape;
    const int64_t BH = static_cast<int64_t>(s.B) * s.Hkv;
    const int32_t page = s.page;
    const int64_t bf16_page_cost = 2LL * page * s.D * 2;            // K + V bytes of a page
    const int64_t slow_row = p->slow_bits == 4 ? s.D / 2 : s.D;       // code bytes per token
    const int64_t i8_page_cost = 2LL * (page * slow_row + page * 4);  // codes + fp32 scales
    const int64_t item_cost = static_cast<int64_t>(p->G) * s.D * 6; // q in + partial out

    struct Chunk {
        int32_t bh, pb, pe, tier_tokens, flags, kv, fl;
        int64_t page_cost;
    };
    std::vector<Chunk> chunks;
    p->planned_kv.assign(static_cast<size_t>(BH), 0);
    int64_t total_pages = 0, kv_bytes = 0;
    for (int64_t bh = 0; bh < BH; ++bh) {
        const int32_t n = kv_len[bh];
        if (n < 0) return TG_EINVAL;
        p->planned_kv[bh] = n;
        const int32_t f = fast_len ? std::max(0, std::min(fast_len[bh], n)) : 0;
        if (fast_len && fast_len[bh] < 0) return TG_EINVAL;
        struct Run { int32_t tokens, flags; int64_t cost; };
        Run runs[2];
        int nr = 0;
        if (fast_len) {
            runs[nr++] = {n - f, kItemSlow, i8_page_cost};
            runs[nr++] = {f, 0, bf16_page_cost};
            kv_bytes += static_cast<int64_t>(n - f) * 2 * (slow_row + 4) + static_cast<int64_t>(f) * 2 * s.D * 2;
        } else {
            runs[nr++] = {n, 0, bf16_page_cost};
            kv_bytes += static_cast<int64_t>(n) * 2 * s.D * 2;
        }
        // pages [0, p0) of a cascade plan's head are read by its cascade units
        const int32_t p0 = pstart ? pstart[bh] : 0;
        int64_t head_pages = 0;
        for (int r = 0; r < nr; ++r) head_pages += (runs[r].tokens + page - 1) / page;
        head_pages -= p0;
        int64_t cap = max_chunk_pages > 0 ? max_chunk_pages : INT32_MAX;
        if (min_splits > 1 && head_pages > 0)
            cap = std::min<int64_t>(cap, std::max<int64_t>(1, head_pages / min_splits));
        for (int r = 0; r < nr; ++r) {
            const int32_t pages = (runs[r].tokens + page - 1) / page - p0;
            if (pages <= 0) continue;
            const int64_t k = (pages + cap - 1) / cap;
            int32_t at = p0;
            for (int64_t c = 0; c < k; ++c) {
                const int32_t sz = static_cast<int32_t>(pages / k + (c < pages % k ? 1 : 0));
                chunks.push_back({static_cast<int32_t>(bh), at, at + sz, runs[r].tokens,
                                  runs[r].flags, n, fast_len ? fast_len[bh] : 0, runs[r].cost});
                at += sz;
            }
            total_pages += pages;
        }
    }
    p->kv_bytes = kv_bytes;

    // Workers: as many as asked, but at least ~8 pages each (tiny batches are not worth the
    // partials and the merge).
    int64_t W = std::max<int64_t>(1, num_workers);
    W = std::max<int64_t>(1, std::min<int64_t>(W, total_pages / 8));
    // Cost of all pages plus one item overhead per (head, tier) run and per worker cut
    // (adjacent chunks of a run on one worker form a single item).
    long double total_cost = static_cast<long double>(W - 1) * item_cost;
    for (size_t i = 0; i < chunks.size(); ++i) {
        const Chunk &c = chunks[i];
        total_cost += static_cast<long double>(c.pe - c.pb) * c.page_cost;
        if (i == 0 || chunks[i - 1].bh != c.bh || chunks[i - 1].flags != c.flags) total_cost += item_cost;
    }

    if (p->whole_heads && !fast_len && !pstart) {
        // Small bf16 batches: every head is one item (no split, so no partials and no merge
        // kernel); heads go to workers longest first, each to the least loaded worker (ties:
        // the lower index), one worker per head at most.
        std::vector<int64_t> heads;
        for (int64_t bh = 0; bh < BH; ++bh)
            if (kv_len[bh] > 0) heads.push_back(bh);
        std::stable_sort(heads.begin(), heads.end(), [&](int64_t x, int64_t y) { return kv_len[x] > kv_len[y]; });
        const int64_t Wh = std::max<int64_t>(1, std::min<int64_t>(std::max(1, num_workers), static_cast<int64_t>(heads.size())));
        std::vector<int64_t> load(static_cast<size_t>(Wh), 0);
        std::vector<std::vector<int64_t>> of(static_cast<size_t>(Wh));
        for (int64_t bh : heads) {
            int64_t w = 0;
            for (int64_t k = 1; k < Wh; ++k)
                if (load[k] < load[w]) w = k;
            load[w] += (kv_len[bh] + page - 1) / page;
            of[w].push_back(bh);
        }
        p->items.clear();
        p->worker_of_item.clear();
        for (int64_t w = 0; w < Wh; ++w)
            for (int64_t bh : of[w]) {
                Item it{};
                it.bh = static_cast<int32_t>(bh);
                it.page_begin = 0;
                it.page_end = (kv_len[bh] + page - 1) / page;
                it.tier_tokens = kv_len[bh];
                it.slot = -1;
                it.flags = 0;
                it.kv_len = kv_len[bh];
                it.fast_len = 0;
                p->items.push_back(it);
                p->worker_of_item.push_back(static_cast<int32_t>(w));
            }
        p->n_workers = p->items.empty() ? 0 : static_cast<int32_t>(Wh);
        p->worker_off.assign(static_cast<size_t>(p->n_workers) + 1, 0);
        for (size_t i = 0; i < p->items.size(); ++i) p->worker_off[p->worker_of_item[i] + 1] = static_cast<int32_t>(i + 1);
        for (int32_t i = 1; i <= p->n_workers; ++i) p->worker_off[i] = std::max(p->worker_off[i], p->worker_off[i - 1]);
        p->dyn_first = static_cast<int32_t>(p->items.size());
        p->n_dyn = 0;
        return finish_slots(p, casc_cnt);
    }

    const bool hybrid = static_permille < 1000;
    const long double sfrac = hybrid ? static_permille / 1000.0L : 1.0L;
    const int32_t dyn_pages = std::max(1, dyn_chunk_pages);
    std::vector<Item> dyn;

    p->items.clear();
    p->worker_of_item.clear();
    int64_t w = 0;
    long double cum = 0;
    auto emit = [&](const Chunk &c, int32_t pb, int32_t pe) {
        // A worker running adjacent chunks of the same head and tier continues the online
        // softmax across them: one item, no partial in between.
        if (!p->items.empty() && p->worker_of_item.back() == static_cast<int32_t>(w)) {
            Item &prev = p->items.back();
            if (prev.bh == c.bh && prev.flags == c.flags && prev.page_end == pb) {
                prev.page_end = pe;
                cum += static_cast<long double>(pe - pb) * c.page_cost;
                return;
            }
        }
        Item it{};
        it.bh = c.bh;
        it.page_begin = pb;
        it.page_end = pe;
        it.tier_tokens = c.tier_tokens;
        it.slot = -1;
        it.flags = c.flags;
        it.kv_len = c.kv;
        it.fast_len = c.fl;
        p->items.push_back(it);
        p->worker_of_item.push_back(static_cast<int32_t>(w));
        cum += static_cast<long double>(pe - pb) * c.page_cost + item_cost;
    };
    // The dynamic region (the cost line after every worker's static share) is collected as
    // spans and cut into dynamic items afterwards.
    struct Span { size_t chunk; int32_t pb, pe; };
    std::vector<Span> dyn_spans;
    auto emit_dyn = [&](const Chunk &c, int32_t pb, int32_t pe) {
        dyn_spans.push_back({static_cast<size_t>(&c - chunks.data()), pb, pe});
    };
    for (const Chunk &c : chunks) {
        int32_t at = c.pb;
        while (at < c.pe) {
            if (hybrid && w == W) { emit_dyn(c, at, c.pe); at = c.pe; break; }
            if (!hybrid && w == W - 1) { emit(c, at, c.pe); at = c.pe; break; }
            const long double target = total_cost * sfrac * static_cast<long double>(w + 1) / W;
            const long double room = target - cum - item_cost;
            const int64_t k = room <= 0 ? 0 : static_cast<int64_t>(room / c.page_cost + 0.5L);
            if (k >= c.pe - at) {
                emit(c, at, c.pe);
                at = c.pe;
            } else if (k >= 1) {
                emit(c, at, at + static_cast<int32_t>(k));
                at += static_cast<int32_t>(k);
                ++w;
            } else {
                ++w;
            }
        }
    }
    // Dynamic items: each span of the dynamic region cut into near-equal pieces of at most
    // dyn_pages pages (pieces never cross a (head, tier) chunk).
    for (const Span &sp : dyn_spans) {
        const Chunk &c = chunks[sp.chunk];
        const int32_t n = sp.pe - sp.pb;
        const int32_t k = (n + dyn_pages - 1) / dyn_pages;
        int32_t at = sp.pb;
        for (int32_t i = 0; i < k; ++i) {
            const int32_t sz = n / k + (i < n % k ? 1 : 0);
            Item it{};
            it.bh = c.bh;
            it.page_begin = at;
            it.page_end = at + sz;
            it.tier_tokens = c.tier_tokens;
            it.slot = -1;
            it.flags = c.flags;
            it.kv_len = c.kv;
            it.fast_len = c.fl;
            dyn.push_back(it);
            at += sz;
        }
    }
    p->n_workers = p->items.empty() ? 0 : p->worker_of_item.back() + 1;
    if (hybrid && !dyn.empty()) p->n_workers = static_cast<int32_t>(W);
    p->worker_off.assign(static_cast<size_t>(p->n_workers) + 1, 0);
    for (size_t i = 0; i < p->items.size(); ++i) p->worker_off[p->worker_of_item[i] + 1] = static_cast<int32_t>(i + 1);
    for (int32_t i = 1; i <= p->n_workers; ++i)
        p->worker_off[i] = std::max(p->worker_off[i], p->worker_off[i - 1]);
    // Dynamic items follow the static ones; they belong to no worker until run time.
    p->dyn_first = static_cast<int32_t>(p->items.size());
    p->n_dyn = static_cast<int32_t>(dyn.size());
    for (const Item &it : dyn) {
        p->items.push_back(it);
        p->worker_of_item.push_back(-1);
    }

    return finish_slots(p, casc_cnt);
}

}  // namespace tg

// ------------------------------------------------------------------------------------------
// Plan creation (host part) and inspection.
// ------------------------------------------------------------------------------------------
namespace {

// Shared-prefix runs of one KV head ("RadixAttention and KV reuse": a radix tree over token
// sequences whose nodes own the KV blocks of their range, reused by every request whose prefix
// passes through the node). Here the tree is recovered from the page tables themselves: the
// rows of head h are grouped by their page id at a position; a group of >= min_readers rows
// that agree on the page forms a node, which runs as far as all of them keep agreeing (full
// pages only); the group is then split again below the node. Each row's private part starts
// where its deepest node ends. Nodes are emitted parent first, groups in order of their first
// row, so the result is deterministic.
struct Node {
    int32_t h, pos_begin, pos_end;
    std::vector<int32_t> readers;
};

void shared_runs(int32_t h, const std::vector<int32_t> &rows, int32_t Hkv, const int32_t *kv_len,
                 const int32_t *table, const int64_t *head_off, int32_t min_readers,
                 std::vector<Node> &nodes, std::vector<int32_t> &pstart) {
    struct Task { std::vector<int32_t> readers; int32_t depth; };
    std::vector<Task> stack;
    stack.push_back({rows, 0});
    auto full = [&](int32_t b) { return kv_len[static_cast<int64_t>(b) * Hkv + h] / 16; };
    auto pid = [&](int32_t b, int32_t pos) {
        return table[head_off[static_cast<int64_t>(b) * Hkv + h] + pos];
    };
    while (!stack.empty()) {
        Task t = std::move(stack.back());
        stack.pop_back();
        std::vector<int32_t> keys;                  // page ids in order of first appearance
        std::vector<std::vector<int32_t>> groups;
        for (int32_t b : t.readers) {
            if (t.depth >= full(b)) continue;
            const int32_t k = pid(b, t.depth);
            size_t gi = 0;
            while (gi < keys.size() && keys[gi] != k) ++gi;
            if (gi == keys.size()) {
                keys.push_back(k);
                groups.emplace_back();
            }
            groups[gi].push_back(b);
        }
        std::vector<Task> children;
        for (size_t gi = 0; gi < groups.size(); ++gi) {
            const std::vector<int32_t> &g = groups[gi];
            if (static_cast<int32_t>(g.size()) < std::max(2, min_readers)) continue;
            int32_t end = t.depth + 1;
            for (;;) {
                bool ok = true;
                for (int32_t b : g)
                    if (end >= full(b) || pid(b, end) != pid(g[0], end)) { ok = false; break; }
                if (!ok) break;
                ++end;
            }
            nodes.push_back({h, t.depth, end, g});
            for (int32_t b : g) pstart[static_cast<int64_t>(b) * Hkv + h] = end;
            children.push_back({g, end});
        }
        for (size_t c = children.size(); c-- > 0;) stack.push_back(std::move(children[c]));
    }
}

// Frees a plan under construction the way tg_plan_destroy does (no CUDA call for a plan that
// holds no device state yet).
struct PlanFree {
    void operator()(tg_plan *p) const { tg_plan_destroy(p); }
};

int plan_create(const tg_shape *shape, const int32_t *kv_len, const int32_t *fast_len,
                const int32_t *group_of_head, const int64_t *group_off, int32_t n_groups,
                int64_t slow_table_len, const tg_plan_opts *opts, const int32_t *table,
                const int64_t *head_off, int64_t table_len, int32_t min_readers, tg_plan **out) {
    if (!out) return TG_EINVAL;
    *out = nullptr;
    if (!shape || !kv_len || !group_of_head || !group_off || n_groups < 1) return TG_EINVAL;
    const tg_shape &s = *shape;
    if (s.B < 0 || s.Hkv < 1 || s.Hq < 1 || s.Hq % s.Hkv != 0 || s.D < 1 || s.page < 1 ||
        s.num_pages < 0 || s.num_slow_pages < 0)
        return TG_EINVAL;
    const int32_t G = s.Hq / s.Hkv;
    if (s.page != 16 || (s.D != 64 && s.D != 128) || (G != 1 && G != 2 && G != 4 && G != 8))
        return TG_EUNSUPPORTED;
    if (fast_len && s.D != 128) return TG_EUNSUPPORTED;
    if (s.num_pages > (INT64_C(1) << 28) || s.num_slow_pages > (INT64_C(1) << 28)) return TG_EUNSUPPORTED;
    if (static_cast<int64_t>(s.B) * s.Hq > INT32_MAX) return TG_EUNSUPPORTED;  // query rows index in 32 bits
    for (int32_t h = 0; h < s.Hkv; ++h)
        if (group_of_head[h] < 0 || group_of_head[h] >= n_groups) return TG_EINVAL;
    const int64_t n_heads = static_cast<int64_t>(s.B) * s.Hkv;
    for (int64_t bh = 0; bh < n_heads; ++bh) {
        if (kv_len[bh] < 0 || (fast_len && fast_len[bh] < 0)) return TG_EINVAL;
        if (kv_len[bh] > TG_MAX_HEAD_TOKENS) return TG_EUNSUPPORTED;
    }
    tg_plan_opts o{};
    o.min_splits = 1;
    o.device = -1;
    if (opts) o = *opts;
    if (o.min_splits < 1) o.min_splits = 1;

    std::unique_ptr<tg_plan, PlanFree> hold(new tg_plan);  // freed on every early return
    tg_plan *p = hold.get();
    p->shape = s;
    p->G = G;
    p->tiered = fast_len != nullptr;
    p->pairs = p->tiered ? tg::kPairsTiered : tg::kPairs;
    p->host_only = o.host_only != 0;
    p->n_groups = n_groups;
    p->slow_table_len = slow_table_len;
    p->group_off.assign(group_off, group_off + n_groups + 1);
    p->device = o.device;
    p->early_prologue = o.early_prologue != 0;
    if (o.wait_limit_us > 0) p->wait_ns = static_cast<uint64_t>(o.wait_limit_us) * 1000ull;
    p->withhold = o.test_withhold_page > 0 ? o.test_withhold_page : 0;
    if (o.capacity && !fast_len) return TG_EINVAL;
    p->capacity = o.capacity != 0;
    p->out_f32 = o.out_f32 != 0;
    p->whole_heads = o.whole_heads != 0;
    p->slow_bits = o.slow_bits == 0 ? 8 : o.slow_bits;
    if ((p->slow_bits != 8 && p->slow_bits != 4) || (p->slow_bits == 4 && (!fast_len || shape->D != 128)))
        return TG_EINVAL;

    // Prefix cascade: shared runs per KV head, cut into units of kCascadeRows query rows.
    std::vector<int32_t> casc_cnt;
    if (table) {
        const int64_t BH = static_cast<int64_t>(s.B) * s.Hkv;
        for (int64_t bh = 0; bh < BH; ++bh) {
            const int64_t npages = (kv_len[bh] + 15) / 16;
            if (kv_len[bh] < 0 || head_off[bh] < 0 || head_off[bh] + npages > table_len) return TG_EINVAL;
        }
        p->pstart.assign(static_cast<size_t>(BH), 0);
        std::vector<Node> nodes;
        std::vector<int32_t> rows(static_cast<size_t>(s.B));
        for (int32_t b = 0; b < s.B; ++b) rows[b] = b;
        for (int32_t h = 0; h < s.Hkv; ++h)
            shared_runs(h, rows, s.Hkv, kv_len, table, head_off, min_readers, nodes, p->pstart);
        casc_cnt.assign(static_cast<size_t>(BH), 0);
        for (const Node &n : nodes)
            for (int32_t b : n.readers) ++casc_cnt[static_cast<int64_t>(b) * s.Hkv + n.h];
        const int32_t per = tg::kCascadeRows / G;
        for (const Node &n : nodes) {
            for (size_t r0 = 0; r0 < n.readers.size(); r0 += per) {
                tg::CascadeUnit u{};
                u.h = n.h;
                u.pos_begin = n.pos_begin;
                u.pos_end = n.pos_end;
                u.n_readers = static_cast<int32_t>(std::min<size_t>(per, n.readers.size() - r0));
                for (int32_t r = 0; r < u.n_readers; ++r) {
                    u.reader[r] = n.readers[r0 + r];
                    u.slot[r] = -1;
                }
                p->cunits.push_back(u);
            }
        }
    }

    int32_t workers = o.num_workers;
    if (!p->host_only) {
        int rc = tg::device_num_sms(o.device, &p->num_sms);
        if (rc != TG_OK) return rc;
        if (workers <= 0) workers = p->num_sms * p->pairs;
    } else if (workers <= 0) {
        workers = 148 * p->pairs;
    }
    const int32_t sp = o.static_permille <= 0 ? 800 : std::min(1000, o.static_permille);
    const int32_t dc = o.dyn_chunk_pages <= 0 ? 16 : o.dyn_chunk_pages;
    int rc = tg::build_work_list(p, kv_len, fast_len, workers, o.min_splits, o.max_chunk_pages, sp,
                                 dc, table ? p->pstart.data() : nullptr,
                                 table ? casc_cnt.data() : nullptr);
    if (rc != TG_OK) return rc;
    if (table) {
        // Cascade partial slots: a head's merge list starts with its runs, in unit order.
        std::vector<int32_t> next(static_cast<size_t>(s.B) * s.Hkv, -1);
        for (const tg::MergeHead &m : p->merge) next[m.bh] = m.first_slot;
        for (tg::CascadeUnit &u : p->cunits)
            for (int32_t r = 0; r < u.n_readers; ++r)
                u.slot[r] = next[static_cast<int64_t>(u.reader[r]) * s.Hkv + u.h]++;
    }
    // Whole-head bf16 plans whose longest head holds at most kLeanMaxPages pages run the lean
    // kernel (one CTA per (sequence, KV head), no copy pipeline to set up): a tiny batch's step
    // is one launch's latency, not bandwidth.
    if (p->whole_heads && !p->tiered && p->cunits.empty()) {
        int64_t most = 0;
        for (const tg::Item &it : p->items) most = std::max<int64_t>(most, it.page_end - it.page_begin);
        p->lean = most <= tg::kLeanMaxPages;
    }
    p->grid = (p->n_workers + p->pairs - 1) / p->pairs;
    if (p->n_dyn > 0 && p->grid == 0) p->grid = 1;
    if (p->grid == 0 && !p->empties.empty()) p->grid = 1;  // the kernel also writes empty heads
    if (!p->host_only) {
        rc = tg::device_init_plan(p);
        if (rc != TG_OK) return rc;
    }
    *out = hold.release();
    return TG_OK;
}

}  // namespace

extern "C" int tg_plan_create(const tg_shape *shape, const int32_t *kv_len,
                              const int32_t *fast_len, const int32_t *group_of_head,
                              const int64_t *group_off, int32_t n_groups,
                              int64_t slow_table_len, const tg_plan_opts *opts,
                              tg_plan **out) {
    return tg::no_throw([&] {
        return plan_create(shape, kv_len, fast_len, group_of_head, group_off, n_groups, slow_table_len, opts,
                           nullptr, nullptr, 0, 0, out);
    });
}

extern "C" int tg_plan_create_cascade(const tg_shape *shape, const int32_t *kv_len,
                                      const int32_t *group_of_head, const int64_t *group_off,
                                      int32_t n_groups, const int32_t *page_table,
                                      const int64_t *head_page_off, int64_t table_len,
                                      int32_t min_readers, const tg_plan_opts *opts,
                                      tg_plan **out) {
    if (out) *out = nullptr;
    if (!page_table || !head_page_off || table_len < 0) return TG_EINVAL;
    return tg::no_throw([&] {
        return plan_create(shape, kv_len, nullptr, group_of_head, group_off, n_groups, 0, opts, page_table,
                           head_page_off, table_len, min_readers, out);
    });
}

extern "C" void tg_plan_destroy(tg_plan *p) {
    if (!p) return;
    if (!p->host_only) tg::device_free_plan(p);
    delete p;
}

extern "C" int tg_plan_get_info(const tg_plan *p, tg_plan_info *info) {
    if (!p || !info) return TG_EINVAL;
    std::memset(info, 0, sizeof(*info));
    info->n_items = static_cast<int64_t>(p->items.size());
    info->n_partials = p->n_partials;
    info->n_merge = static_cast<int64_t>(p->merge.size());
    info->n_empty = static_cast<int64_t>(p->empties.size());
    info->n_dynamic = p->n_dyn;
    info->n_workers = p->n_workers;
    info->grid = p->lean ? static_cast<int32_t>(static_cast<int64_t>(p->shape.B) * p->shape.Hkv) : p->grid;
    info->block = p->lean ? tg::kLeanWarps * 32 : p->pairs * 64;
    info->smem_bytes = p->lean ? 0 : p->smem_bytes;
    info->stages = p->lean ? 0 : p->stages;
    info->device_bytes = p->dev_bytes;
    info->kv_bytes = p->kv_bytes;
    info->n_cascade = static_cast<int32_t>(p->cunits.size());
    return TG_OK;
}

extern "C" int tg_plan_cascade_units(const tg_plan *p, int32_t *units) {
    if (!p || !units) return TG_EINVAL;
    const int32_t w = 4 + 2 * tg::kCascadeRows;
    for (size_t i = 0; i < p->cunits.size(); ++i) {
        const tg::CascadeUnit &u = p->cunits[i];
        int32_t *o = units + static_cast<int64_t>(w) * static_cast<int64_t>(i);
        o[0] = u.h; o[1] = u.pos_begin; o[2] = u.pos_end; o[3] = u.n_readers;
        for (int32_t r = 0; r < tg::kCascadeRows; ++r) {
            o[4 + r] = r < u.n_readers ? u.reader[r] : -1;
            o[4 + tg::kCascadeRows + r] = r < u.n_readers ? u.slot[r] : -1;
        }
    }
    return TG_OK;
}

extern "C" int tg_plan_items(const tg_plan *p, int32_t *items) {
    if (!p || !items) return TG_EINVAL;
    for (size_t i = 0; i < p->items.size(); ++i) {
        const tg::Item &it = p->items[i];
        int32_t *o = items + 8 * i;
        o[0] = it.bh; o[1] = it.page_begin; o[2] = it.page_end; o[3] = it.tier_tokens;
        o[4] = it.slot; o[5] = it.flags & tg::kItemSlow; o[6] = p->worker_of_item[i];
        o[7] = it.slot >= 0 ? (it.flags >> 1) : -1;
    }
    return TG_OK;
}
