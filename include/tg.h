/*
 * tg.h — C ABI of the B200 ragged / prefix-shared / tiered paged decode library (libtg.so).
 *
 * One decode step of attention for a batch of sequences whose KV cache is paged, where every
 * (sequence, KV head) keeps its own number of tokens:
 *   - per-head budgets fixed at admission and ragged page tables grouped by budget
 *     ("Tangram" explainer, arXiv 2606.06302: 核心方法 / 三大机制 1 Budget Reservation,
 *     2 Ragged Paging, 3 Ahead-of-Time Load Balancing);
 *   - prefix pages shared across sequences through their page tables (RadixAttention lesson,
 *     Phase 17 · 06: the radix tree as KV index and its worked example);
 *   - a recent bf16 tier and an older INT8 or INT4 tier dequantised inside the attention loop
 *     (HBM-resident, or streamed block-wise from host memory)
 *     ("TTKV" explainer, arXiv 2604.19769: 核心方法 1 Tier Layout, 2 Tier Content,
 *     3 Tier Interaction);
 *   - split-K over each head's tokens merged by log-sum-exp (CAP survey, arXiv 2405.11299,
 *     §2.4.3 "加速单个请求": the online normaliser; Fig. 5 Dist Attention).
 *
 * Conventions for every function:
 *   - Return value: TG_OK (0) or one of the TG_E* codes below. Nothing throws across the ABI
 *     (one exception, stated at tg_plan_timing_enable); host allocation failures return
 *     TG_ENOMEM and leave the objects as they were.
 *   - Host pointers are read during the call only. Device pointers are caller-owned device
 *     memory (allocate them with any allocator); the library never frees them.
 *   - Device calls are stream-ordered and asynchronous on the given stream; they allocate
 *     nothing, synchronise nothing and re-plan nothing per call. Pass the stream as the
 *     cudaStream_t value cast to tg_stream (NULL = legacy default stream).
 *   - Layouts are row-major and contiguous unless stated. "bf16" = IEEE bfloat16 bits.
 *   - Device base pointers must be 16-byte aligned (TG_EINVAL otherwise).
 *   - Query head hq uses KV head hq / (Hq/Hkv) (contiguous GQA groups of G = Hq/Hkv).
 *   - Supported by the kernels: page = 16 tokens, D in {64, 128}, G in {1, 2, 4, 8};
 *     the tiered kernel needs D = 128. Other shapes return TG_EUNSUPPORTED.
 *   - Not thread-safe per object: one host thread at a time per tg_alloc / tg_plan.
 */
#ifndef TG_H
#define TG_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TG_OK 0
#define TG_EINVAL 1        /* bad argument: null/misaligned pointer, inconsistent sizes */
#define TG_ENOSPC 2        /* page pool exhausted; the allocator state is unchanged */
#define TG_EBADPAGE 3      /* a kernel met a page id outside the pool, a table row outside its
                              group table, or lengths that differ from the plan; the offending
                              pages were skipped (never read), the affected rows are unspecified */
#define TG_ECUDA 4         /* a CUDA runtime call failed (message via tg_last_cuda_error) */
#define TG_ETIMEOUT 5      /* a kernel wait exceeded its bound; the kernel returned early */
#define TG_ENOMEM 6        /* host or device allocation failed */
#define TG_ENOTFOUND 7     /* unknown sequence or segment id */
#define TG_EUNSUPPORTED 8  /* shape outside what the kernels support */
#define TG_EEXIST 9        /* sequence id already holds a reservation */

/* Longest retained length of one (sequence, KV head) that plans accept (2^30 tokens, 2^26
 * pages): every token and page index of a head then fits 32-bit arithmetic with room to spare. */
#define TG_MAX_HEAD_TOKENS (1 << 30)

typedef struct CUstream_st *tg_stream; /* == cudaStream_t */

/* Shape of one decode step over one layer. */
typedef struct tg_shape {
    int32_t B;              /* sequences */
    int32_t Hq;             /* query heads */
    int32_t Hkv;            /* KV heads; Hq % Hkv == 0 */
    int32_t D;              /* head dimension */
    int32_t page;           /* tokens per page (16) */
    int32_t reserved;       /* 0 */
    int64_t num_pages;      /* pages in the bf16 pools (k_pages, v_pages / k_fast, v_fast) */
    int64_t num_slow_pages; /* pages in the INT8 / INT4 pools (tiered decode only; else 0) */
} tg_shape;

/* Human-readable text of a status code (static storage). */
const char *tg_strerror(int status);
/* Text of the last CUDA error seen by this library on the calling thread ("" if none). */
const char *tg_last_cuda_error(void);

/* =====================================================================================
 * Host-side admission steps (pure host code; no device needed).
 * ===================================================================================== */

/* Retained length from the budget table ("Tangram" 关键发现: per-head retention ratios from
 * an input-invariant head ranking; 三大机制 1: footprint fixed at admission).
 * For i < n: kv_len[i] = 0 if full_len[i] <= 0, else
 *   min(full_len[i], max(1, floor((ratio_ppm[i] * full_len[i] + 500000) / 1000000))).
 * ratio_ppm in [0, 1000000]; out of range -> TG_EINVAL. Arrays host, length n. */
int tg_retained_lengths(int64_t n, const int32_t *full_len, const int32_t *ratio_ppm,
                        int32_t *kv_len);

/* Budget groups ("Tangram" 三大机制 2, Ragged Paging: heads with similar budgets share one
 * page table). Heads ranked by budget ascending (ties by index); rank p of n_heads goes to
 * group floor(p * n_groups / n_heads). budget_ppm, group_of_head: host, length n_heads.
 * 1 <= n_groups <= n_heads, else TG_EINVAL. */
int tg_budget_groups(int32_t n_heads, const int32_t *budget_ppm, int32_t n_groups,
                     int32_t *group_of_head);

/* ---- Budget-reservation page allocator ("Tangram" 三大机制 1; RadixAttention worked
 * example for shared segments). A FIFO free list of page ids: reservations take pages from
 * the front, releases append freed pages at the back in release order. Owns only host
 * memory. */
typedef struct tg_alloc tg_alloc;

/* Allocator over a pool of num_pages pages (>= 1) of `page` tokens each (>= 1) whose initial
 * free list is a seeded shuffle of the page ids (the pool's pages in no particular order, as a
 * long-running server's pool): the Fisher-Yates (Durstenfeld) shuffle of 0..num_pages-1 that
 * for i = num_pages-1 down to 1 swaps entries i and (x_k mod (i+1)), where x_0, x_1, ... is the
 * SplitMix64 sequence seeded with `seed` (Steele, Lea & Flood 2014: state += 0x9E3779B97F4A7C15,
 * output = its 64-bit finaliser) and k counts the swaps from 0. */
int tg_alloc_create(int64_t num_pages, int32_t page, uint64_t seed, tg_alloc **out);
/* As tg_alloc_create with the initial free-list order given: free_order is a permutation of
 * 0..num_pages-1 (NULL = ascending). A non-permutation returns TG_EINVAL. */
int tg_alloc_create_ordered(int64_t num_pages, int32_t page, const int32_t *free_order,
                            tg_alloc **out);
void tg_alloc_destroy(tg_alloc *a);
int64_t tg_alloc_free_pages(const tg_alloc *a);   /* pages currently on the free list */
/* References held on a page (0 = free; a shared page counts its segment plus each reader). */
int32_t tg_alloc_refcount(const tg_alloc *a, int32_t page_id);

/* Shared segment of n_tokens tokens for n_heads KV heads: floor(n_tokens/page) full pages per
 * head, taken head ascending, page ascending. Only full pages are shared; a partial tail goes
 * into each reader's private pages. *seg_id receives the segment id; page_ids (may be NULL)
 * receives [n_heads][floor(n_tokens/page)]. All-or-nothing: TG_ENOSPC leaves state unchanged. */
int tg_share_segment(tg_alloc *a, int32_t n_tokens, int32_t n_heads, int32_t *seg_id,
                     int32_t *page_ids);

/* Reservation of sequence seq_id at admission: for each KV head h (ascending), its page list
 * is the full pages of each segment in prefix_segs[0..n_prefix) (in order; a negative id is
 * skipped), followed by ceil((kv_len[h] - shared tokens)/page) private pages from the free
 * list. kv_len[h] must be >= the shared tokens (TG_EINVAL otherwise). All-or-nothing:
 * TG_ENOSPC leaves state unchanged. page_ids (host, capacity entries) receives the lists
 * head after head; head_count (host, n_heads entries, may be NULL) each head's page count
 * (its shared pages plus its private ones), the head_count rows tg_build_group_tables takes;
 * *n_written (may be NULL) the total. Each head's count is ceil(kv_len[h]/page) when every
 * shared segment holds whole pages. seq_id must be new (TG_EEXIST). */
int tg_reserve(tg_alloc *a, int32_t seq_id, int32_t n_heads, const int32_t *kv_len,
               int32_t n_prefix, const int32_t *prefix_segs, int32_t *page_ids,
               int64_t capacity, int32_t *head_count, int64_t *n_written);
/* Release a sequence: private pages return to the free list, shared pages drop one reference. */
int tg_release(tg_alloc *a, int32_t seq_id);
/* Drop a segment's own reference; its pages return once no sequence reads them. */
int tg_release_segment(tg_alloc *a, int32_t seg_id);

/* Group page tables ("Tangram" 三大机制 2). For B sequences x Hkv heads with head_count[b][h]
 * pages whose ids are listed in page_ids (flat: b ascending, h ascending, page ascending —
 * the order tg_reserve writes them for b = 0, 1, ...): group g's table is dense
 * [B][H_g][P_g] (heads of g ascending, P_g = max page count in g, unused slots -1); tables
 * concatenated in group order. Writes head_off[B*Hkv] (start of each row) and
 * group_off[n_groups+1] (start of each group table; group_off[n_groups] = total length).
 * table may be NULL to query the length (head_off then may be NULL too); otherwise it must
 * hold group_off[n_groups] entries. All arrays host. */
int tg_build_group_tables(int32_t B, int32_t Hkv, const int32_t *head_count,
                          const int32_t *group_of_head, int32_t n_groups,
                          const int32_t *page_ids, int32_t *table, int64_t *head_off,
                          int64_t *group_off);

/* Ahead-of-time placement of sequences on GPUs ("Tangram" 三大机制 3): longest-processing-
 * time greedy over seq_bytes (descending, ties by index) onto the least-loaded GPU (ties by
 * lowest index). gpu_of_seq: host, length n_seq. */
int tg_place_sequences(int32_t n_seq, const int64_t *seq_bytes, int32_t n_gpus,
                       int32_t *gpu_of_seq);

/* =====================================================================================
 * Plan: the static work list of one layer's decode step (single-GPU form of "Tangram"
 * 三大机制 3: balanced ahead of time, never re-planned per step).
 * ===================================================================================== */
typedef struct tg_plan tg_plan;

typedef struct tg_plan_opts {
    int32_t num_workers;      /* 0: (SM count) x (workers per CTA) of the device */
    int32_t min_splits;       /* cut every head into at least this many chunks (>= 1) */
    int32_t max_chunk_pages;  /* 0: no cap; else chunks hold at most this many pages */
    int32_t host_only;        /* 1: build the work list on the host only (inspection, or
                                 tg_ragged_paged_decode_noalloc; the other decode calls reject
                                 such a plan); 0: also create device state */
    int32_t device;           /* CUDA device ordinal, -1 = current */
    int32_t static_permille;  /* share of the bytes assigned to workers ahead of time, in
                                 1/1000 (0 = default 800; 1000 = all static); the rest is
                                 cut into dynamic items that workers take in order */
    int32_t dyn_chunk_pages;  /* pages per dynamic item, at most (0 = default 16) */
    int32_t early_prologue;   /* decode kernels are launched as programmatic dependents (CUDA
                                 programmatic dependent launch) of the preceding kernel in the
                                 stream. 0 (default): they wait for it before doing anything.
                                 1: before waiting they already read this plan and the page
                                 tables, head offsets, lengths and group map; queries, K/V and
                                 every output are touched only after the wait. Use 1 only if no
                                 preceding kernel that triggers its dependents early writes
                                 those tables (this library's own kernels never do). */
    int32_t wait_limit_us;    /* bound of any single wait inside the decode kernel, in µs
                                 (0 = default 4 s); a wait that runs out stops the kernel and
                                 the call reports TG_ETIMEOUT through tg_plan_status */
    int32_t test_withhold_page; /* testing only (0 = off): worker 0's producer never signals
                                 its page number test_withhold_page (1-based), so a bounded
                                 wait runs out on purpose; no copy is issued for that page */
    int32_t capacity;         /* tiered plans only ("TTKV" tiers that grow every step): 1 = the
                                 kv_len / fast_len given to tg_plan_create are capacities, the
                                 reserved slots of each head (fast tier: fast_len; INT8 tier:
                                 kv_len - fast_len); each decode call reads the current lengths
                                 from head_kv_len / head_fast_len (which must fit them, else
                                 TG_EBADPAGE) and skips reserved pages that hold no token yet,
                                 so appends (tg_tiered_append) never need a new plan. 0: the
                                 lengths are exact, as for bf16 plans */
    int32_t out_f32;          /* 1: the decode calls' out is fp32 [B][Hq][D] (the normalised
                                 output before bf16 rounding, e.g. a partial result to be merged
                                 with others by tg_lse_merge); 0 (default): bf16 */
    int32_t slow_bits;        /* tiered plans: code width of the slow tier, 8 (0 = default) or
                                 4 (D = 128 only): INT4 pools are uint8 [num_slow_pages][16][D/2]
                                 as tg_quantize_int4 writes them, passed where the INT8 calls
                                 take k_q8 / v_q8 */
    int32_t whole_heads;      /* bf16 plans without a cascade: 1 = every head is one item (no
                                 split heads, so no partials and no merge kernel), for small
                                 batches, where a step is launch-bound. When no head holds more
                                 than 64 pages the plan runs the lean kernel: one CTA per
                                 (sequence, KV head) reading its pages with plain 16-byte loads
                                 (no copy pipeline, no tensor map, no shared-memory ring), fp32
                                 scores and probabilities, one launch per call (the H2O scores
                                 call keeps the pipelined kernel; the lean kernel records no
                                 worker timeline). Otherwise whole heads are placed on up to
                                 num_workers workers longest first. Ignored for tiered and
                                 cascade plans; static_permille, min_splits and max_chunk_pages
                                 do not apply */
} tg_plan_opts;

/* Build a plan. kv_len[B*Hkv] (host): retained tokens per (sequence, KV head); the decode
 * calls check the device copy against it. fast_len[B*Hkv] (host) or NULL: tiered plan whose
 * last min(fast_len, kv_len) tokens of each head are in the bf16 tier and the rest in the slow
 * tier (INT8, or INT4 with opts->slow_bits = 4). group_of_head[Hkv] and group_off[n_groups+1] (host; from tg_budget_groups /
 * tg_build_group_tables) bound every row of the bf16 (fast) table to its group table; for a tiered
 * plan slow_table_len bounds the slow tier's table (ignored otherwise).
 * Each head's tokens are cut into chunks (min_splits, max_chunk_pages; chunks never cross a
 * tier boundary). The first static_permille of the chunks' byte cost is partitioned into
 * num_workers equal contiguous ranges assigned ahead of time (at least ~8 pages per worker;
 * fewer workers for tiny batches); the rest is cut into dynamic items of at most
 * dyn_chunk_pages pages that workers take from a shared ticket when their own range is done
 * (absorbing per-SM bandwidth differences). A head cut into several items is merged by
 * log-sum-exp in split order by a second kernel that the decode call launches as a
 * programmatic dependent (its launch overlaps the decode's tail).
 * The plan owns one device allocation (work list, merge list, partial results, error word),
 * made here; nothing is allocated per call. Returns TG_EINVAL for bad arguments (a negative
 * length among them), TG_EUNSUPPORTED for a shape the kernels do not serve (page != 16, D not
 * 64 or 128, Hq/Hkv not 1, 2, 4 or 8, a tiered plan with D != 128, a kv_len above
 * TG_MAX_HEAD_TOKENS, B*Hq above INT32_MAX), TG_ENOMEM when host or device memory runs out; on any error *out is
 * NULL and nothing is left allocated. */
int tg_plan_create(const tg_shape *shape, const int32_t *kv_len, const int32_t *fast_len,
                   const int32_t *group_of_head, const int64_t *group_off, int32_t n_groups,
                   int64_t slow_table_len, const tg_plan_opts *opts, tg_plan **out);
void tg_plan_destroy(tg_plan *p);

typedef struct tg_plan_info {
    int64_t n_items;          /* work items */
    int64_t n_partials;       /* items that write a partial result (heads with > 1 item) */
    int64_t n_merge;          /* heads split over several items (merged by the merge kernel) */
    int64_t n_empty;          /* heads with no retained token (out = 0, lse = -inf) */
    int64_t n_dynamic;        /* items taken from the shared ticket at run time */
    int32_t n_workers;        /* workers that have items */
    int32_t grid;             /* CTAs of the decode kernel */
    int32_t block;            /* threads per CTA */
    int32_t smem_bytes;       /* dynamic shared memory per CTA */
    int32_t stages;           /* pipeline stages per worker */
    int32_t n_cascade;        /* prefix-cascade units (tg_plan_create_cascade), else 0 */
    int64_t device_bytes;     /* bytes of the plan's device allocation */
    int64_t kv_bytes;         /* retained K/V bytes one step reads (scales included) */
} tg_plan_info;
int tg_plan_get_info(const tg_plan *p, tg_plan_info *info);

/* Prefix-aware cascade plan for shared pages ("RadixAttention and KV reuse": a radix tree over
 * token sequences, each node owning the KV blocks of its range, reused by every request whose
 * prefix passes through it). As tg_plan_create (bf16, no tiers), and from the HOST copies of the
 * page table and head offsets (page_table int32 [table_len], head_page_off int64 [B*Hkv]) it
 * recovers, per KV head, the runs of full pages that >= min_readers (at least 2) heads' rows
 * share at the same positions: rows are grouped by their page id at a position, a group runs
 * as far as all its rows keep the same page ids, then splits again below. Every run is read
 * once per step by cascade units of up to 256 query rows (256/G readers with their G query
 * heads each: two 128-row tiles for tcgen05.mma, S and O in tensor memory) instead of once per
 * reader; each reader's
 * private pages (after its deepest run) go through the ordinary split-K items; every head with
 * a run is merged from its run partials (in run order) and its items'. Results equal those of
 * tg_ragged_paged_decode up to rounding; the plan stays valid while the device table and
 * lengths are the ones given here. TG_EINVAL on a row outside the table. */
int tg_plan_create_cascade(const tg_shape *shape, const int32_t *kv_len,
                           const int32_t *group_of_head, const int64_t *group_off,
                           int32_t n_groups, const int32_t *page_table,
                           const int64_t *head_page_off, int64_t table_len, int32_t min_readers,
                           const tg_plan_opts *opts, tg_plan **out);
/* Inspection: per cascade unit (tg_plan_info.n_cascade of them), 4 + 2*256 ints: KV head, first
 * page position, end page position, readers, then 256 reader sequences and 256 partial slots
 * (-1 past the readers). */
int tg_plan_cascade_units(const tg_plan *p, int32_t *units);

/* Work list export for inspection: items (host, n_items x 8 int32): per item
 * {b*Hkv + h, page_begin, page_end, tier_tokens, partial slot (-1 = final), INT8 tier (0/1),
 * worker (-1 = dynamic), merge-list index (-1 = final)}; page indices are within the head's
 * row of its tier's table. */
int tg_plan_items(const tg_plan *p, int32_t *items);

/* Read and clear the plan's device error word after the work queued on stream: returns
 * TG_OK, TG_EBADPAGE or TG_ETIMEOUT. Synchronises the stream (a debugging aid). After a
 * timeout it also resets the split heads' arrival tickets, so the plan can be used again. */
int tg_plan_status(tg_plan *p, tg_stream stream);

/* Kernel timing (a profiling aid). With max_calls > 0, the next max_calls decode calls on this
 * plan record CUDA events on their stream before the decode kernel, between it and the merge
 * kernel, and after the merge kernel (a recorded call gives up the merge kernel's launch
 * overlap); later calls record nothing. The events are created here (no device memory);
 * max_calls = 0 destroys them. tg_plan_timing_read waits for the last recorded event, returns
 * the number of calls recorded and the summed decode-kernel and merge-kernel times in
 * milliseconds, and restarts the count. The host table of 3 * max_calls events is the one
 * allocation in this library whose failure is not turned into TG_ENOMEM (std::bad_alloc
 * propagates): keep max_calls to what the caller means to time (the bench uses <= 256). */
int tg_plan_timing_enable(tg_plan *p, int32_t max_calls);
int tg_plan_timing_read(tg_plan *p, int32_t *n_calls, double *decode_ms, double *merge_ms);

/* Worker timeline (a profiling aid). With on = 1 the plan allocates n_workers x 8 uint64
 * device words (here, not per call) and every later decode call records, per worker: the
 * global timer (ns) at CTA start, first copy issued, first page ready, stop marker seen and
 * worker done; then the number of dynamic items it took; words 6 and 7 are written as zero
 * (split heads are merged by the merge kernel, after the decode kernel). tg_plan_trace_read
 * synchronises the stream and copies the last call's words to trace (host, n_workers x 8).
 * on = 0 frees the buffer. */
int tg_plan_trace_enable(tg_plan *p, int32_t on);
int tg_plan_trace_read(tg_plan *p, uint64_t *trace, tg_stream stream);

/* =====================================================================================
 * Decode entry points (device).
 * ===================================================================================== */

/* Ragged paged decode ("Tangram" 三大机制 2 Ragged Paging; CAP §2.4.3 online normaliser):
 * for every query row (b, hq), h = hq / G, n = head_kv_len[b*Hkv+h], the retained tokens
 * t < n are read through the page table (page = page_table[head_page_off[b*Hkv+h] + t/16],
 * slot t % 16) and
 *   lse = ln sum_t exp(s_t),  s_t = scale * q . K_t,   out = sum_t exp(s_t - lse) V_t.
 * n = 0 gives out = 0, lse = -inf.
 *   plan        from tg_plan_create with fast_len = NULL and this shape.
 *   q           device bf16 [B][Hq][D]
 *   k_pages     device bf16 [num_pages][16][D];   v_pages likewise
 *   page_table  device int32, the concatenated group tables (tg_build_group_tables)
 *   head_page_off device int64 [B*Hkv];  head_kv_len device int32 [B*Hkv] (must equal the
 *               plan's kv_len); group_of_head device int32 [Hkv]
 *   scale       softmax scale applied in fp32 (e.g. 1/sqrt(D))
 *   out         device bf16 [B][Hq][D];  lse device fp32 [B][Hq] (natural log)
 * One kernel launch: reads each page once with the Tensor Memory Accelerator; computes q.K
 * and P.V on tensor cores (bf16 in, fp32 accumulate; P rounded to bf16); heads covered by one
 * item write out/lse directly; split heads write one partial per item, and a second kernel
 * (a programmatic dependent launch, so its launch overlaps the decode's tail) merges them by
 * log-sum-exp in split order, so results are deterministic. */
int tg_ragged_paged_decode(tg_plan *plan, const void *q, const void *k_pages,
                           const void *v_pages, const int32_t *page_table,
                           const int64_t *head_page_off, const int32_t *head_kv_len,
                           const int32_t *group_of_head, float scale, void *out, float *lse,
                           tg_stream stream);

/* tg_ragged_paged_decode that also writes every retained token's scores for the H2O rule
 * below: token_scores (device fp32, 4-byte aligned, [table_len*16][G]) gets, at entry
 * (head_page_off[b*Hkv+h]*16 + t)*G + g, s = scale * q[b][h*G+g] . K_t (natural-log units, as
 * computed for the softmax) for every retained t < head_kv_len; other entries are untouched.
 * Costs 4*G bytes of writes per retained token. */
int tg_ragged_paged_decode_scores(tg_plan *plan, const void *q, const void *k_pages,
                                  const void *v_pages, const int32_t *page_table,
                                  const int64_t *head_page_off, const int32_t *head_kv_len,
                                  const int32_t *group_of_head, float scale, void *out, float *lse,
                                  float *token_scores, tg_stream stream);

/* Ragged paged decode that allocates no device memory. The source pages have no counterpart:
 * this entry exists for callers that cannot allocate device memory after start-up — an engine
 * that reserves the whole device for its KV pool and treats any later cudaMalloc as a failure,
 * a plug-in whose host framework owns every device allocation, a runtime that permits
 * allocation only during initialisation. Arguments and results are those of
 * tg_ragged_paged_decode; plan may be a host-only plan (tg_plan_opts.host_only = 1), which holds
 * no device memory (the one case where a decode call accepts a host-only plan; cascade plans
 * return TG_EUNSUPPORTED). A plan made for a device (tg_plan_opts.device >= 0) runs only on
 * that device (TG_EINVAL when another one is current); a host-only plan made with device -1
 * runs on the current device. The kernels' scratch (the plan's work list, copied in by plain
 * host-to-device copies on the stream, and the split heads' partial results) lives in one
 * fixed 16 MiB device array inside this library, which every GPU that loads the library holds
 * until the process exits; a plan that needs more returns TG_ENOMEM (the message says how much
 * it needs) without launching anything. The first call on a device also looks up the array's
 * device address, clears its error word and sets the kernels' shared-memory limit on that
 * device; make that first call before any stream capture. All calls share the array and each
 * call overwrites it: calls whose work overlaps on the GPU (other streams, other host threads)
 * race and must be serialised by the caller. The plan's wait bound (wait_limit_us) applies.
 * Kernel-side range errors are skipped as in the plan-based entry and, with timeouts, are
 * recorded in the array's error word, read by tg_ragged_paged_decode_noalloc_status. Calls no
 * cudaMalloc, cudaFree or allocating library routine. */
int tg_ragged_paged_decode_noalloc(tg_plan *plan, const void *q, const void *k_pages,
                                   const void *v_pages, const int32_t *page_table,
                                   const int64_t *head_page_off, const int32_t *head_kv_len,
                                   const int32_t *group_of_head, float scale, void *out,
                                   float *lse, tg_stream stream);
/* Read and clear the error word of tg_ragged_paged_decode_noalloc's array on the current device,
 * after the work queued on stream: TG_OK, TG_EBADPAGE or TG_ETIMEOUT for the no-alloc calls
 * since the last read (TG_OK if no such call has run on this device). Synchronises the stream;
 * allocates nothing. */
int tg_ragged_paged_decode_noalloc_status(tg_stream stream);

/* Tiered decode ("TTKV" 核心方法 1-3): as tg_ragged_paged_decode over the union of two tiers.
 * Per head, f = min(head_fast_len, n): tokens [0, n - f) are in the INT8 tier (row starts at
 * slot 0 of slow_page_table[slow_head_off[b*Hkv+h]]), tokens [n - f, n) in the bf16 tier
 * (row starts at slot 0 of fast_page_table[fast_head_off[b*Hkv+h]]).
 *   k_q8, v_q8       device int8 [num_slow_pages][16][D] (symmetric codes)
 *   k_scale, v_scale device fp32 [num_slow_pages][16] (per token per head): K_t = code * scale
 *   k_fast, v_fast   device bf16 [num_pages][16][D]
 * INT8 K codes enter an integer tensor-core product against q written per row as two int8
 * digits, q = s_q (q1 + q2/254) (|error| <= max|q| / 64516 per element), exact in int32; INT8
 * V codes are converted exactly to fp16 in registers; the K scale multiplies the score and the
 * V scale multiplies the probability before P.V (both in fp32). plan from tg_plan_create with
 * this fast_len. D must be 128. Plans with tg_plan_opts.slow_bits = 4 read an INT4 tier here
 * instead (k_q8 / v_q8 then point to packed uint8 [num_slow_pages][16][D/2] pools of
 * tg_quantize_int4): its K nibbles enter the same product (unsigned, offset corrected in
 * int32), its V nibbles are widened exactly to fp16. */
int tg_tiered_decode(tg_plan *plan, const void *q, const int8_t *k_q8, const int8_t *v_q8,
                     const float *k_scale, const float *v_scale, const int32_t *slow_page_table,
                     const int64_t *slow_head_off, const void *k_fast, const void *v_fast,
                     const int32_t *fast_page_table, const int64_t *fast_head_off,
                     const int32_t *head_kv_len, const int32_t *head_fast_len, float scale,
                     void *out, float *lse, tg_stream stream);

/* =====================================================================================
 * Host-buffer decode pipeline (no counterpart on the pages: the decode step as a serving loop
 * calls it, queries arriving in and outputs leaving through host memory). A pipe owns two
 * device staging sets (q, out, lse of a plan's shape) and two copy streams (host->device,
 * device->host). Call i uses set i % 2: its input copy waits until call i-2's decode has read
 * that set; its decode runs on `stream` after that copy and after call i-2's output copy; its
 * output copy follows its decode. So the copies of neighbouring calls overlap this call's
 * decode, and calls return at once. Host buffers must be page-locked (cudaHostAlloc or
 * cudaHostRegister; pageable memory makes the copies synchronous); q_host must stay unchanged
 * and out_host / lse_host unread until tg_host_pipe_wait (or a tg_host_pipe_join'd stream)
 * says the call is done.
 * ===================================================================================== */
typedef struct tg_host_pipe tg_host_pipe;

/* Create a pipe for calls on plans of `plan`'s shape (B, Hq, D) and device. Allocates
 * 2 x (2 B*Hq*D*2 + B*Hq*4) bytes of device memory, two streams and six events.
 * TG_EINVAL for a host-only plan or one with tg_plan_opts.out_f32 (the pipe carries bf16
 * outputs; calls with such a plan are rejected too); TG_ENOMEM; TG_ECUDA. */
int tg_host_pipe_create(const tg_plan *plan, tg_host_pipe **out);
/* Wait for the pipe's copies, then free it. NULL is ignored. */
void tg_host_pipe_destroy(tg_host_pipe *p);
/* Block the host until every copy issued on the pipe has finished (all out / lse delivered). */
int tg_host_pipe_wait(tg_host_pipe *p);
/* Device-side ordering with another stream: tg_host_pipe_after makes the pipe's copy streams
 * wait for the work queued on `stream` so far; tg_host_pipe_join makes `stream` wait for every
 * copy issued on the pipe so far (e.g. to bracket a run of calls between two events). */
int tg_host_pipe_after(tg_host_pipe *p, tg_stream stream);
int tg_host_pipe_join(tg_host_pipe *p, tg_stream stream);

/* tg_ragged_paged_decode / tg_tiered_decode with q_host (bf16 [B][Hq][D]) read from host
 * memory and out_host (bf16 [B][Hq][D]) / lse_host (fp32 [B][Hq]) written to host memory
 * through the pipe; every other argument as in those calls. TG_EINVAL if the plan's shape or
 * device differs from the pipe's or a host pointer is NULL; otherwise the decode call's
 * status. */
int tg_ragged_paged_decode_host(tg_host_pipe *p, tg_plan *plan, const void *q_host,
                                const void *k_pages, const void *v_pages,
                                const int32_t *page_table, const int64_t *head_page_off,
                                const int32_t *head_kv_len, const int32_t *group_of_head,
                                float scale, void *out_host, float *lse_host, tg_stream stream);
int tg_tiered_decode_host(tg_host_pipe *p, tg_plan *plan, const void *q_host,
                          const int8_t *k_q8, const int8_t *v_q8, const float *k_scale,
                          const float *v_scale, const int32_t *slow_page_table,
                          const int64_t *slow_head_off, const void *k_fast, const void *v_fast,
                          const int32_t *fast_page_table, const int64_t *fast_head_off,
                          const int32_t *head_kv_len, const int32_t *head_fast_len, float scale,
                          void *out_host, float *lse_host, tg_stream stream);

/* =====================================================================================
 * TTKV slow tier in host memory, streamed block-wise ("TTKV" 核心方法 1 Tier Layout: the slow
 * tier in DRAM, the fast tier in HBM; 3 Tier Interaction: Block-wise Streaming Attention, the
 * DRAM data fetched in blocks with the fetch overlapping the computation). The INT8 pool (codes
 * int8 [num_slow_pages][16][D] for K and V, scales fp32 [num_slow_pages][16]) stays in
 * page-locked host memory. Its pages are cut into blocks of block_pages consecutive page ids;
 * each block that holds a retained token is copied per step into one of ring_blocks HBM slots
 * (copy stream) and decoded when it lands (compute stream) while the next block copies. Each
 * block and the bf16 fast tier give an fp32 partial per query row; one merge kernel combines
 * them by log-sum-exp (fast tier first, then blocks in page order). Results equal
 * tg_tiered_decode's up to rounding.
 * ===================================================================================== */
typedef struct tg_slow_stream tg_slow_stream;

/* Build the per-block tables and plans (host) and, unless opts->host_only, the device state:
 * the ring (ring_blocks x block_pages pages of codes and scales), the block tables, partials
 * fp32 [1 + blocks][B*Hq][D + 1], a copy stream and 2 x ring_blocks events. Arguments as
 * tg_plan_create for a tiered plan (kv_len, fast_len, group_of_head, group_off, n_groups over
 * the fast tier's group tables) plus the INT8 tier's HOST table (slow_page_table int32
 * [slow_table_len], slow_head_off int64 [B*Hkv]); shape->num_slow_pages = pages of the host pool.
 * opts as for tg_plan_create (out_f32 and capacity are set by the stream); with
 * opts->slow_bits = 4 the host pool holds packed INT4 codes, uint8 [num_slow_pages][16][D/2]
 * as tg_quantize_int4 writes them, and the ring is sized for them. Returns TG_EINVAL on a bad
 * argument or a page id outside the pool, TG_EUNSUPPORTED for a kv_len above
 * TG_MAX_HEAD_TOKENS, TG_ENOMEM when host or device memory runs out; *out is NULL on error. */
int tg_slow_stream_create(const tg_shape *shape, const int32_t *kv_len, const int32_t *fast_len,
                          const int32_t *group_of_head, const int64_t *group_off,
                          int32_t n_groups, const int32_t *slow_page_table,
                          const int64_t *slow_head_off, int64_t slow_table_len,
                          int32_t block_pages, int32_t ring_blocks, const tg_plan_opts *opts,
                          tg_slow_stream **out);
/* Wait for the stream's copies, then free it. NULL is ignored. */
void tg_slow_stream_destroy(tg_slow_stream *s);
/* Inspection: returns the number of streamed blocks J (blocks with no retained token are
 * skipped) and, for non-NULL arrays, each block's first page id (int64 [J]), its page count
 * (int32 [J]) and the tokens of every (sequence, KV head) in it (int32 [J][B*Hkv]). */
int tg_slow_stream_blocks(const tg_slow_stream *s, int64_t *first_page, int32_t *pages,
                          int32_t *tokens);
/* The worst device status over the stream's plans (as tg_plan_status; synchronises). */
int tg_slow_stream_status(tg_slow_stream *s, tg_stream stream);

/* One tiered decode step with the INT8 tier read from page-locked HOST memory (k_q8_host,
 * v_q8_host, k_scale_host, v_scale_host; pageable memory is rejected with TG_EINVAL). q, the
 * fast tier (k_fast, v_fast bf16 pools, fast_page_table, fast_head_off, group_of_head) and
 * out (bf16 [B][Hq][D]) / lse (fp32 [B][Hq]) are device buffers, as for tg_tiered_decode; the
 * lengths are the ones given to tg_slow_stream_create. Stream-ordered: the copies start after
 * the work already queued on `stream`, and out / lse are complete when `stream` reaches the
 * end of the call. */
int tg_tiered_decode_streamed(tg_slow_stream *s, const void *q, const int8_t *k_q8_host,
                              const int8_t *v_q8_host, const float *k_scale_host,
                              const float *v_scale_host, const void *k_fast, const void *v_fast,
                              const int32_t *fast_page_table, const int64_t *fast_head_off,
                              const int32_t *group_of_head, float scale, void *out, float *lse,
                              tg_stream stream);

/* Log-sum-exp merge of split results (CAP §2.4.3 online normaliser; Fig. 5 Dist Attention):
 * for each of n_rows rows, its splits j = row_split_off[r] .. row_split_off[r+1]-1 hold a
 * normalised partial part_o[j][D] (fp32) and part_lse[j] (fp32, natural log):
 *   lse = ln sum_j exp(part_lse[j]),  out = sum_j exp(part_lse[j] - lse) part_o[j]
 * in split order; a row with no splits (or only -inf splits) gets out = 0, lse = -inf.
 * All pointers device; row_split_off int64 [n_rows+1]; out bf16 [n_rows][D]; lse fp32. */
int tg_lse_merge(int64_t n_rows, int32_t D, const int64_t *row_split_off, const float *part_o,
                 const float *part_lse, void *out, float *lse, tg_stream stream);

/* INT8 slow-tier quantisation ("TTKV" 核心方法 1/3: older tokens stored quantised; scheme
 * left open by the page): per row (token of one head) of D bf16 values,
 *   amax = max |x|, scale = amax / 127 (fp32), code = clamp(rint(x / scale), -127, 127)
 * with an IEEE fp32 quotient and ties to even; amax = 0 gives scale 0 and zero codes.
 * src device bf16 [n_rows][D]; codes device int8 [n_rows][D]; scale device fp32 [n_rows].
 * A page of the INT8 pool is 16 consecutive rows. */
int tg_quantize_int8(int64_t n_rows, int32_t D, const void *src, int8_t *codes, float *scale,
                     tg_stream stream);

/* INT4 slow-tier quantisation ("TTKV" 核心方法 1 Tier Layout names INT8 or INT4 for the slow
 * tier; the scheme is left open): the INT8 rule with 7 levels a side,
 *   scale = amax / 7 (fp32), code = clamp(rint(x / scale), -7, 7),
 * packed two codes per byte as offset-binary nibbles: byte i (i < D/2) of a row is
 * (code_i + 8) | (code_{i+D/2} + 8) << 4. src device bf16 [n_rows][D]; packed device uint8
 * [n_rows][D/2]; scale device fp32 [n_rows]. Tiered plans with slow_bits = 4 read this layout. */
int tg_quantize_int4(int64_t n_rows, int32_t D, const void *src, uint8_t *packed, float *scale,
                     tg_stream stream);

/* =====================================================================================
 * Decode-step write path ("Tangram" 三大机制 1 Budget Reservation and 落地形态; CAP §2.4.1
 * (3) static and (4) dynamic sparsity of decoder-only models).
 * A head's footprint is fixed when its request starts: head_budget[b*Hkv+h] slots, laid out
 * like the retained tokens (slot t in page page_table[head_page_off[b*Hkv+h] + t/16], row
 * t % 16; the caller reserved ceil(budget/16) pages). head_kv_len counts the slots in use,
 * 0 .. kv_len-1. A decode step appends one token per (sequence, KV head): a head with a free
 * slot takes it (kv_len grows by one); a full head overwrites one retained token and keeps
 * kv_len = budget, so no page is ever reclaimed or added. Per-slot metadata (slot_pos,
 * slot_score) is indexed by table position: entry head_page_off[b*Hkv+h]*16 + t.
 * Common arguments: shape (B, Hq, Hkv, D with D % 8 == 0, page = 16, num_pages); k_new, v_new
 * device bf16 [B][Hkv][D], 16-byte aligned: the step's new rows; k_pages, v_pages the bf16
 * pool (written); slot_out device int32 [B*Hkv]: the slot written, or -1 when nothing was
 * written (budget < 1, or the table's page id outside [0, num_pages)). All device pointers;
 * calls are stream-ordered and allocate nothing. Returns TG_EINVAL on a null/misaligned
 * pointer or bad shape, TG_ECUDA on a launch error.
 * ===================================================================================== */

/* Static rule (LM-Infinite / StreamingLLM): keep the first s = min(sink, budget-1) positions of
 * the sequence and the budget - s most recent. A full head overwrites slot s + cursor and
 * advances cursor modulo budget - s; head_cursor (int32 [B*Hkv], in/out) is 0 for a head whose
 * retained tokens sit in slots in position order, sinks first. One launch, one warp per head;
 * moves 4*D bytes per head. */
int tg_append_sink_recent(const tg_shape *shape, int32_t sink, const void *k_new,
                          const void *v_new, void *k_pages, void *v_pages,
                          const int32_t *page_table, const int64_t *head_page_off,
                          const int32_t *head_budget, int32_t *head_kv_len, int32_t *head_cursor,
                          int32_t *slot_out, tg_stream stream);

/* Score-based rule (H2O), append half: a full head overwrites slot head_victim[b*Hkv+h] (int32
 * [B*Hkv], from tg_h2o_update; ignored while the head has a free slot, which is taken
 * instead); the written slot's slot_pos (int32, in/out) becomes new_pos[b] (int32 [B]) and its
 * slot_score (fp32, in/out) 0. One launch, one warp per head. */
int tg_append_h2o(const tg_shape *shape, const void *k_new, const void *v_new, void *k_pages,
                  void *v_pages, const int32_t *page_table, const int64_t *head_page_off,
                  const int32_t *head_budget, int32_t *head_kv_len, const int32_t *head_victim,
                  int32_t *slot_pos, float *slot_score, const int32_t *new_pos,
                  int32_t *slot_out, tg_stream stream);

/* Score-based rule (H2O), bookkeeping half, run after a decode step: each retained token's
 * score grows by the attention the step's G query heads paid it,
 *   slot_score += sum_g exp(token_scores[entry][g] - lse[b][h*G+g])
 * (token_scores from tg_ragged_paged_decode_scores, lse from the same call; token_scores =
 * NULL skips this), then head_victim[b*Hkv+h] gets the slot the next token takes: kv_len while
 * the head has a free slot; else, among tokens older than the last `recent` positions
 * (slot_pos < next_pos[b] - recent), the lowest score (ties: lowest slot); if every token is
 * recent, the oldest one; -1 for budget < 1. One launch, one CTA per head; reads 8 + 4*G bytes
 * and writes 4 per retained token. */
int tg_h2o_update(const tg_shape *shape, int32_t recent, const float *token_scores,
                  const float *lse, const int64_t *head_page_off, const int32_t *head_budget,
                  const int32_t *head_kv_len, const int32_t *slot_pos, float *slot_score,
                  const int32_t *next_pos, int32_t *head_victim, tg_stream stream);

/* Tier migration ("TTKV" 核心方法 1 Tier Layout, 2 Tier Content: the most recent tokens stay in
 * the high-precision fast tier, older ones move to the quantised slow tier). Per (sequence, KV
 * head): the fast tier holds the last f = head_fast_len tokens of the n = head_kv_len, at most
 * head_fast_cap of them, token at position p in fast slot p mod head_fast_cap of its fast row
 * (fast_page_table / fast_head_off, as for tg_tiered_decode); the INT8 tier holds positions
 * [0, n - f) at slow index = position (slow_page_table / slow_head_off; head_slow_cap reserved
 * slots). Appending position n: with f < cap (then n == f: every token is still fast) it takes
 * fast slot n; with a full window the oldest fast token (position n - cap) is quantised into
 * slow index n - cap with the rule of tg_quantize_int8 (codes and scale bit-exact with it) and
 * the new token takes its fast slot. head_kv_len grows by one, head_fast_len up to the cap.
 *   k_new, v_new  device bf16 [B][Hkv][D] (16-byte aligned); k_fast, v_fast the bf16 pools;
 *   k_q8, v_q8, k_scale, v_scale the INT8 pools and scales (written); shape.num_pages and
 *   shape.num_slow_pages bound the page ids; D % 32 == 0, D <= 128.
 *   moved_out (int32 [B*Hkv]): slow index written, or -1; slot_out: fast slot written, or -1
 *   when nothing was appended (a state outside the rules above, no reserved slow slot left, or
 *   a page id outside its pool).
 * One launch, one warp per head. A tiered plan made with tg_plan_opts.capacity = 1 for the
 * reserved sizes decodes every later state without a new plan. */
int tg_tiered_append(const tg_shape *shape, const void *k_new, const void *v_new, void *k_fast,
                     void *v_fast, const int32_t *fast_page_table, const int64_t *fast_head_off,
                     const int32_t *head_fast_cap, int8_t *k_q8, int8_t *v_q8, float *k_scale,
                     float *v_scale, const int32_t *slow_page_table, const int64_t *slow_head_off,
                     const int32_t *head_slow_cap, int32_t *head_kv_len, int32_t *head_fast_len,
                     int32_t *moved_out, int32_t *slot_out, tg_stream stream);

/* tg_tiered_append into an INT4 slow tier: the leaving token is quantised with the rule of
 * tg_quantize_int4 (scale = amax / 7; codes and scale bit-exact with it) into the packed
 * pools k_q4, v_q4 (uint8 [num_slow_pages][16][D/2], byte i = d i low nibble and d i + D/2
 * high nibble, offset-binary); everything else as tg_tiered_append. Tiered plans with
 * tg_plan_opts.slow_bits = 4 (and capacity = 1) decode the result. */
int tg_tiered_append_int4(const tg_shape *shape, const void *k_new, const void *v_new,
                          void *k_fast, void *v_fast, const int32_t *fast_page_table,
                          const int64_t *fast_head_off, const int32_t *head_fast_cap,
                          uint8_t *k_q4, uint8_t *v_q4, float *k_scale, float *v_scale,
                          const int32_t *slow_page_table, const int64_t *slow_head_off,
                          const int32_t *head_slow_cap, int32_t *head_kv_len,
                          int32_t *head_fast_len, int32_t *moved_out, int32_t *slot_out,
                          tg_stream stream);

/* =====================================================================================
 * SplitZip: lossless BF16 codec for KV transfer ("SplitZip" explainer, arXiv 2605.01708, "Die
 * SplitZip-Strategie", "Warum es schnell ist"). A bf16 value is sign, 8-bit exponent and 7-bit
 * mantissa; the 16 most frequent exponents get 4-bit codes, two per byte; rare exponents go to
 * an escape stream (position, exponent) applied as overwrites on decode. Stream layout:
 *   codebook uint8[16]: exponents by count descending, ties by exponent ascending (over all
 *            256, so always 16 distinct entries);
 *   sm       uint8[n]: (sign << 7) | mantissa;  (16-byte aligned)
 *   codes    uint8[(n+1)/2]: element i's code in byte i/2, low nibble for even i; an escaped
 *            element carries code 0;  (8-byte aligned)
 *   esc_pos  int64[esc_cap], esc_exp uint8[esc_cap]: escapes in ascending position; n_esc (one
 *            device int64) their number — if it exceeds esc_cap the stream is incomplete.
 * All pointers device; calls are stream-ordered and allocate nothing.
 * ===================================================================================== */

/* Bytes of device workspace tg_splitzip_encode needs for n elements: about n/8 + 12 KB. The
 * workspace must be 256-byte aligned. Returns -1 for n < 0. */
int64_t tg_splitzip_workspace_bytes(int64_t n);

/* Encode n bf16 values (src, 16-byte aligned). Kernels: exponent histogram, codebook, a
 * 4096-element tile per CTA writing sm and codes (and, in tiles that hold escapes, which
 * elements escape), and one escape pass that places each tile's escapes at its offset.
 * Errors: TG_EINVAL for negative sizes, null or misaligned pointers; TG_ECUDA on a launch
 * failure (tg_last_cuda_error() has the text). */
int tg_splitzip_encode(int64_t n, const void *src, uint8_t *codebook, uint8_t *sm,
                       uint8_t *codes, int64_t *esc_pos, uint8_t *esc_exp, int64_t esc_cap,
                       int64_t *n_esc, void *workspace, tg_stream stream);

/* Decode into dst (bf16 [n], 16-byte aligned): codes through the codebook, then the escapes. */
int tg_splitzip_decode(int64_t n, const uint8_t *codebook, const uint8_t *sm,
                       const uint8_t *codes, const int64_t *esc_pos, const uint8_t *esc_exp,
                       const int64_t *n_esc, int64_t esc_cap, void *dst, tg_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* TG_H */
