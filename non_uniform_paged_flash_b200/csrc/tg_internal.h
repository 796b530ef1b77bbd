// Internal declarations shared by the host library (tg_host.cpp) and the CUDA side
// (tg_kernels.cu) of libtg. Not part of the ABI.
#pragma once

#include <cstdint>
#include <new>
#include <stdexcept>
#include <string>
#include <vector>

#include "tg.h"

namespace tg {

// The host code builds std containers. A C entry point runs its body through no_throw so that
// a container that cannot grow (std::bad_alloc, or a length past its limit) returns TG_ENOMEM
// instead of unwinding through the C ABI. Bodies make their fallible allocations before they
// change any state that outlives the call.
template <class F>
int no_throw(F &&body) noexcept {
    try {
        return body();
    } catch (const std::bad_alloc &) {
        return TG_ENOMEM;
    } catch (const std::length_error &) {
        return TG_ENOMEM;
    }
}

// One work item: a contiguous page range of one (sequence, KV head) row in one tier.
struct Item {
    int32_t bh;          // b * Hkv + h
    int32_t page_begin;  // first page (index within the head's row of its tier's table)
    int32_t page_end;    // one past the last page
    int32_t tier_tokens; // tokens held by this head's row in this tier (tail-page mask)
    int32_t slot;        // partial-result slot, -1 = this item writes the final output
    int32_t flags;       // bit 0 kItemSlow (INT8 tier); bits 1.. merge-list index
    int32_t kv_len;      // planned retained length of the head (checked on device)
    int32_t fast_len;    // planned fast-tier length (tiered plans), else 0
};
static_assert(sizeof(Item) == 32, "Item is 32 bytes");
constexpr int32_t kItemSlow = 1;

// A head split over nsplit >= 2 consecutive partial slots, merged after the decode kernel.
struct MergeHead {
    int32_t bh;
    int32_t first_slot;
    int32_t nsplit;
    int32_t pad;
};

// Prefix cascade: one unit = up to 256 query rows (two tensor-core tiles of 128; kCascadeRows / G
// readers, each with its G query heads) that read the same run of shared pages
// [pos_begin, pos_end) of KV head h: the pages are identical in every reader's table row. Each
// reader gets one partial result.
constexpr int kCascadeRows = 256;
struct CascadeUnit {
    int32_t h;
    int32_t pos_begin;  // first page position (index within every reader's row)
    int32_t pos_end;    // one past the last
    int32_t n_readers;
    int32_t reader[kCascadeRows];  // sequence b of each reader
    int32_t slot[kCascadeRows];    // partial-result slot of (b, h) for this run
};
static_assert(sizeof(CascadeUnit) == 16 + 8 * kCascadeRows, "CascadeUnit layout");

// Device error-word bits.
constexpr uint32_t kErrBadPage = 1u;   // page id outside the pool
constexpr uint32_t kErrBadRow = 2u;    // row outside its group table / table
constexpr uint32_t kErrPlan = 4u;      // device lengths differ from the plan
constexpr uint32_t kErrTimeout = 8u;   // a bounded wait gave up

// Launch geometry of the decode kernels (see tg_kernels.cu): (producer warp, consumer warp)
// pairs per CTA. The tiered kernel's INT8 consumer is latency-bound, so it trades ring depth
// for consumers (measured: 6 pairs with 4 stages beat 4 x 6, 7 x 3 and 8 x 3).
constexpr int kPairs = 4;              // bf16 decode kernel
constexpr int kPairsTiered = 6;        // tiered decode kernel (12 warps; 4 ring stages at D = 128)
constexpr int kThreads = kPairs * 64;  // threads per CTA of the bf16 decode kernel
constexpr int kTraceWords = 8;         // worker timeline words (see tg_plan_trace_enable)
// Lean decode kernel (whole-head bf16 plans of short heads: tiny batches where a step is one
// launch's latency): one CTA of kLeanWarps warps per (sequence, KV head), for heads of at most
// kLeanMaxPages pages.
constexpr int kLeanWarps = 8;
constexpr int kLeanMaxPages = 64;

}  // namespace tg

struct tg_plan {
    tg_shape shape{};
    int32_t G = 0;
    bool tiered = false;
    bool host_only = true;
    int device = 0;
    int num_sms = 0;
    int32_t n_groups = 0;
    int64_t slow_table_len = 0;

    // host copies
    std::vector<tg::Item> items;
    std::vector<int32_t> worker_of_item;
    std::vector<int32_t> worker_off;  // [n_workers + 1] (static items)
    int32_t dyn_first = 0;            // dynamic items: items[dyn_first ..]
    int32_t n_dyn = 0;
    std::vector<tg::MergeHead> merge;
    std::vector<int32_t> empties;     // heads with no retained token
    std::vector<int64_t> group_off;   // [n_groups + 1]
    std::vector<int32_t> planned_kv;  // [B*Hkv]
    std::vector<tg::CascadeUnit> cunits;  // prefix cascade units (cascade plans only)
    std::vector<int32_t> pstart;          // [B*Hkv] first page of the head's private part
    int64_t n_partials = 0;
    int32_t merge_warps = 1;          // warps per (split head, row) CTA of the merge kernel
    int32_t pairs = tg::kPairs;       // worker pairs per CTA of this plan's decode kernel
    bool early_prologue = false;      // see tg_plan_opts.early_prologue
    uint64_t wait_ns = 4000000000ull; // bound of any single wait in the decode kernel
    int32_t withhold = 0;             // see tg_plan_opts.test_withhold_page
    bool capacity = false;            // see tg_plan_opts.capacity
    bool out_f32 = false;             // see tg_plan_opts.out_f32
    int32_t slow_bits = 8;            // see tg_plan_opts.slow_bits
    bool whole_heads = false;         // see tg_plan_opts.whole_heads
    bool lean = false;                // whole-head plan run by the lean kernel (short heads)
    int32_t n_workers = 0;
    int64_t kv_bytes = 0;

    // launch geometry
    int32_t grid = 0;
    int32_t stages = 0;
    int32_t stage_bytes = 0;
    int32_t smem_bytes = 0;

    // device state: one allocation carved into these
    void *dev_base = nullptr;
    int64_t dev_bytes = 0;
    tg::Item *d_items = nullptr;
    int32_t *d_worker_off = nullptr;
    tg::MergeHead *d_merge = nullptr;
    int64_t *d_group_off = nullptr;
    float *d_part_o = nullptr;    // [n_partials][G][D]
    float *d_part_lse = nullptr;  // [n_partials][G]
    int32_t *d_empties = nullptr;   // [n_empty]
    uint32_t *d_dyn = nullptr;      // [2] dynamic ticket, producers done
    tg::CascadeUnit *d_cunits = nullptr;
    int32_t *d_planned = nullptr;   // [B*Hkv] planned lengths (lean plans)
    uint32_t *d_err = nullptr;

    // kernel timing: 2 events per recorded call (cudaEvent_t stored as void*)
    std::vector<void *> tev;
    int32_t tev_cap = 0;
    int32_t tev_count = 0;
    uint64_t *d_trace = nullptr;  // worker timeline, n_workers x kTraceWords (when enabled)

    // tensor-map cache keyed by the pool pointers of the last call
    const void *tm_key[4] = {nullptr, nullptr, nullptr, nullptr};
    alignas(64) unsigned char tmaps[4][128];
};

namespace tg {
// Host planner (tg_host.cpp): fills items / worker_off / merge / n_partials / kv_bytes.
// pstart (nullable): first page of each head's private part (earlier pages are covered by
// cascade units); casc_cnt (nullable): the head's cascade partials, merged before its items.
int build_work_list(tg_plan *p, const int32_t *kv_len, const int32_t *fast_len,
                    int32_t num_workers, int32_t min_splits, int32_t max_chunk_pages,
                    int32_t static_permille, int32_t dyn_chunk_pages,
                    const int32_t *pstart = nullptr, const int32_t *casc_cnt = nullptr);
// Device side (tg_kernels.cu).
int device_init_plan(tg_plan *p);
void device_free_plan(tg_plan *p);
int device_num_sms(int device, int *num_sms);
void set_cuda_error(const char *what, int code);
}  // namespace tg
