// TTKV slow tier in host memory, streamed block-wise ("TTKV" 核心方法 1 Tier Layout: the slow
// tier lives in DRAM; 3 Tier Interaction: Block-wise Streaming Attention — DRAM data is fetched
// in blocks and the fetch overlaps the computation). The INT8 pool stays in page-locked host
// memory. Contiguous blocks of its pages are copied into a ring of HBM slots on a copy stream;
// each block is decoded as it lands by a tiered plan over that block's pages (fp32 partial per
// query row), the bf16 fast tier by a plan of its own, and one merge kernel combines the
// partials by log-sum-exp. Copies and decodes are ordered by events only:
//   block j, slot r = j % ring:  copy:    wait freed[r]; host pages -> slot r; record landed[r]
//                                compute: wait landed[r]; decode block j; record freed[r]
// so the copy of block j+1 runs while block j is decoded.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <memory>
#include <new>
#include <vector>

#include "tg.h"
#include "tg_internal.h"

struct tg_slow_stream {
    tg_shape shape{};
    int device = 0;
    int32_t G = 0;
    int32_t block_pages = 0, ring = 0;
    int32_t row_bytes = 0;                  // code bytes per token and tensor: D (INT8) or D/2 (INT4)
    bool host_only = true;
    tg_plan *fast = nullptr;                // bf16 plan over the fast tier (fp32 out)
    std::vector<tg_plan *> blk;             // one tiered plan per streamed block (fp32 out)
    std::vector<int64_t> blk_first;         // first host page of each streamed block
    std::vector<int32_t> blk_pages;         // pages copied for each block
    std::vector<int32_t> blk_len;           // [n_blocks][B*Hkv] tokens of each head in each block
    std::vector<int64_t> blk_table_len;     // per block
    std::vector<int64_t> blk_table_base;    // per block: its table's start within h_table
    std::vector<int32_t> h_table;           // all blocks' tables, concatenated
    std::vector<int64_t> h_off;             // [n_blocks][B*Hkv] row starts within the block's table
    // device
    void *dev = nullptr;
    int8_t *ring_k = nullptr, *ring_v = nullptr;
    float *ring_ks = nullptr, *ring_vs = nullptr;
    int32_t *d_table = nullptr, *d_len = nullptr, *d_zero = nullptr, *d_fast_len = nullptr;
    int64_t *d_off = nullptr;
    float *part_o = nullptr, *part_lse = nullptr;  // [1 + n_blocks][B*Hq][D], [1 + n_blocks][B*Hq]
    cudaStream_t copy = nullptr;
    std::vector<cudaEvent_t> landed, freed;
    cudaEvent_t start = nullptr;
};

namespace tg {
namespace {

// One warp per query row: out = sum_j exp(lse_j - lse) o_j, lse = ln sum_j exp(lse_j), over
// the parts in order (fast tier first, then the blocks).
template <int D>
__global__ void __launch_bounds__(256) stream_merge_kernel(int32_t parts, int64_t rows, const float *po,
                                                           const float *pl, __nv_bfloat16 *out, float *lse) {
    constexpr int VEC = D / 32;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    float m = -INFINITY, sum = 0.f, acc[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) acc[c] = 0.f;
    for (int j = 0; j < parts; ++j) {
        const float l = pl[static_cast<int64_t>(j) * rows + r];
        if (l == -INFINITY) continue;
        const float mn = fmaxf(m, l);
        const float a = m == -INFINITY ? 0.f : expf(m - mn), w = expf(l - mn);
        const float *o = po + (static_cast<int64_t>(j) * rows + r) * D + lane * VEC;
        sum = sum * a + w;
#pragma unroll
        for (int c = 0; c < VEC; ++c) acc[c] = acc[c] * a + w * o[c];
        m = mn;
    }
    const float inv = m == -INFINITY ? 0.f : 1.f / sum;
#pragma unroll
    for (int c = 0; c < VEC; ++c) out[r * D + lane * VEC + c] = __float2bfloat16_rn(acc[c] * inv);
    if (lane == 0) lse[r] = m == -INFINITY ? -INFINITY : m + logf(sum);
}

int fail(const char *what, cudaError_t e) {
    set_cuda_error(what, static_cast<int>(e));
    return TG_ECUDA;
}

size_t a256(size_t b) { return (b + 255) / 256 * 256; }

void release(tg_slow_stream *s) {
    if (s->fast) tg_plan_destroy(s->fast);
    for (tg_plan *p : s->blk) tg_plan_destroy(p);
    for (cudaEvent_t e : s->landed) cudaEventDestroy(e);
    for (cudaEvent_t e : s->freed) cudaEventDestroy(e);
    if (s->start) cudaEventDestroy(s->start);
    if (s->copy) cudaStreamDestroy(s->copy);
    if (s->dev) cudaFree(s->dev);
    delete s;
}

bool pinned(const void *p) {
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeHost;
}

}  // namespace
}  // namespace tg

using namespace tg;

namespace {

struct Release {
    void operator()(tg_slow_stream *s) const { release(s); }
};

int slow_stream_create(const tg_shape *shape, const int32_t *kv_len, const int32_t *fast_len,
                       const int32_t *group_of_head, const int64_t *group_off, int32_t n_groups,
                       const int32_t *slow_page_table, const int64_t *slow_head_off, int64_t slow_table_len,
                       int32_t block_pages, int32_t ring_blocks, const tg_plan_opts *opts, tg_slow_stream **out) {
    if (!out) return TG_EINVAL;
    *out = nullptr;
    if (!shape || !kv_len || !fast_len || !group_of_head || !group_off || !slow_head_off ||
        block_pages < 1 || ring_blocks < 1 || slow_table_len < 0 || shape->B < 1 || shape->Hkv < 1 ||
        shape->Hq < shape->Hkv || shape->Hq % shape->Hkv || shape->page != 16 ||
        (shape->D != 64 && shape->D != 128) || shape->num_slow_pages < 0 || (slow_table_len > 0 && !slow_page_table))
        return TG_EINVAL;
    tg_plan_opts o{};
    if (opts) o = *opts;
    const tg_shape &S = *shape;
    const int64_t BH = static_cast<int64_t>(S.B) * S.Hkv;
    const int64_t nsp = S.num_slow_pages;
    block_pages = static_cast<int32_t>(std::min<int64_t>(block_pages, std::max<int64_t>(1, nsp)));  // no slot beyond the pool
    const int64_t n_all_blocks = (nsp + block_pages - 1) / block_pages;

    // Rows of each block: a head's pages that fall in the block, its partial tail page last.
    std::vector<int32_t> fl(static_cast<size_t>(BH));
    std::vector<std::vector<int32_t>> rows(static_cast<size_t>(n_all_blocks * BH));
    std::vector<int32_t> tail(static_cast<size_t>(n_all_blocks * BH), 0);
    for (int64_t bh = 0; bh < BH; ++bh) {
        const int32_t n = kv_len[bh];
        if (n < 0 || fast_len[bh] < 0) return TG_EINVAL;
        if (n > TG_MAX_HEAD_TOKENS) return TG_EUNSUPPORTED;
        const int32_t f = std::min(fast_len[bh], n);
        fl[bh] = f;
        const int32_t ns = n - f;
        const int32_t np = (ns + 15) / 16;
        if (np > 0 && (slow_head_off[bh] < 0 || slow_head_off[bh] > slow_table_len - np)) return TG_EINVAL;
        for (int32_t t = 0; t < np; ++t) {
            const int32_t id = slow_page_table[slow_head_off[bh] + t];
            if (id < 0 || id >= nsp) return TG_EINVAL;
            const int64_t j = id / block_pages;
            const int32_t local = static_cast<int32_t>(id - j * block_pages);
            const bool is_tail = t == np - 1 && ns % 16 != 0;
            if (is_tail) tail[j * BH + bh] = (ns % 16) | (local << 8);  // tokens | page << 8
            else rows[j * BH + bh].push_back(local);
        }
    }
    std::unique_ptr<tg_slow_stream, Release> hold(new tg_slow_stream());  // released on every early return
    tg_slow_stream *s = hold.get();
    s->shape = S;
    s->G = S.Hq / S.Hkv;
    s->block_pages = block_pages;
    s->ring = ring_blocks;
    s->row_bytes = o.slow_bits == 4 ? S.D / 2 : S.D;
    s->host_only = o.host_only != 0;
    for (int64_t j = 0; j < n_all_blocks; ++j) {
        bool used = false;
        for (int64_t bh = 0; bh < BH && !used; ++bh) used = !rows[j * BH + bh].empty() || tail[j * BH + bh];
        if (!used) continue;  // no page of this block holds a token: it is never copied
        s->blk_first.push_back(j * block_pages);
        s->blk_pages.push_back(static_cast<int32_t>(std::min<int64_t>(block_pages, nsp - j * block_pages)));
        int64_t at = 0;
        s->blk_table_base.push_back(static_cast<int64_t>(s->h_table.size()));
        for (int64_t bh = 0; bh < BH; ++bh) {
            const std::vector<int32_t> &r = rows[j * BH + bh];
            s->h_off.push_back(at);
            for (int32_t id : r) s->h_table.push_back(id);
            int32_t len = static_cast<int32_t>(r.size()) * 16;
            if (tail[j * BH + bh]) {
                s->h_table.push_back(tail[j * BH + bh] >> 8);
                len += tail[j * BH + bh] & 0xFF;
            }
            s->blk_len.push_back(len);
            at += static_cast<int64_t>(r.size()) + (tail[j * BH + bh] ? 1 : 0);
        }
        s->blk_table_len.push_back(at);
    }
    const int64_t J = static_cast<int64_t>(s->blk_first.size());

    // Plans: the fast tier (bf16, lengths min(fast_len, kv_len)) and one tiered plan per block
    // whose every token is in the INT8 tier; all write fp32 partials.
    tg_plan_opts po = o;
    po.out_f32 = 1;
    po.capacity = 0;
    tg_shape fs = S;
    fs.num_slow_pages = 0;
    tg_plan_opts fo = po;
    fo.slow_bits = 0;
    s->blk.reserve(static_cast<size_t>(J));  // so that keeping a made plan never throws
    int rc = tg_plan_create(&fs, fl.data(), nullptr, group_of_head, group_off, n_groups, 0, &fo, &s->fast);
    std::vector<int32_t> zeros(static_cast<size_t>(BH), 0);
    tg_shape bs = S;
    bs.num_slow_pages = block_pages;
    for (int64_t j = 0; j < J && rc == TG_OK; ++j) {
        tg_plan *p = nullptr;
        rc = tg_plan_create(&bs, s->blk_len.data() + j * BH, zeros.data(), group_of_head, group_off, n_groups,
                            std::max<int64_t>(1, s->blk_table_len[j]), &po, &p);
        if (rc == TG_OK) s->blk.push_back(p);
    }
    if (rc != TG_OK) return rc;
    if (s->host_only) {
        *out = hold.release();
        return TG_OK;
    }

    // Device state: ring | tables | offsets | lengths | zeros | fast lengths | partials.
    std::vector<int32_t> lens(s->blk_len);
    lens.insert(lens.end(), zeros.begin(), zeros.end());
    lens.insert(lens.end(), fl.begin(), fl.end());
    s->landed.reserve(static_cast<size_t>(ring_blocks));
    s->freed.reserve(static_cast<size_t>(ring_blocks));
    s->device = s->fast->device;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(s->device);
    const size_t D = static_cast<size_t>(S.D);
    const size_t slot_codes = static_cast<size_t>(block_pages) * 16 * static_cast<size_t>(s->row_bytes);
    const size_t slot_scales = static_cast<size_t>(block_pages) * 16 * sizeof(float);
    const size_t rows_q = static_cast<size_t>(S.B) * static_cast<size_t>(S.Hq);
    const size_t parts = static_cast<size_t>(1 + J);
    size_t off[9];
    size_t at = 0;
    const size_t sizes[9] = {a256(ring_blocks * slot_codes), a256(ring_blocks * slot_codes),
                             a256(ring_blocks * slot_scales), a256(ring_blocks * slot_scales),
                             a256(std::max<size_t>(1, s->h_table.size()) * 4), a256(s->h_off.size() * 8 + 8),
                             a256((s->blk_len.size() + 2 * static_cast<size_t>(BH)) * 4),
                             a256(parts * rows_q * D * 4), a256(parts * rows_q * 4)};
    for (int i = 0; i < 9; ++i) {
        off[i] = at;
        at += sizes[i];
    }
    cudaError_t e = cudaMalloc(&s->dev, at);
    if (e != cudaSuccess) {
        cudaSetDevice(prev);
        return e == cudaErrorMemoryAllocation ? TG_ENOMEM : fail("cudaMalloc(slow stream)", e);
    }
    char *b = static_cast<char *>(s->dev);
    s->ring_k = reinterpret_cast<int8_t *>(b + off[0]);
    s->ring_v = reinterpret_cast<int8_t *>(b + off[1]);
    s->ring_ks = reinterpret_cast<float *>(b + off[2]);
    s->ring_vs = reinterpret_cast<float *>(b + off[3]);
    s->d_table = reinterpret_cast<int32_t *>(b + off[4]);
    s->d_off = reinterpret_cast<int64_t *>(b + off[5]);
    s->d_len = reinterpret_cast<int32_t *>(b + off[6]);
    s->d_zero = s->d_len + s->blk_len.size();
    s->d_fast_len = s->d_zero + BH;
    s->part_o = reinterpret_cast<float *>(b + off[7]);
    s->part_lse = reinterpret_cast<float *>(b + off[8]);
    if ((!s->h_table.empty() &&
         (e = cudaMemcpy(s->d_table, s->h_table.data(), s->h_table.size() * 4, cudaMemcpyHostToDevice)) != cudaSuccess) ||
        (!s->h_off.empty() &&
         (e = cudaMemcpy(s->d_off, s->h_off.data(), s->h_off.size() * 8, cudaMemcpyHostToDevice)) != cudaSuccess) ||
        (e = cudaMemcpy(s->d_len, lens.data(), lens.size() * 4, cudaMemcpyHostToDevice)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&s->copy, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&s->start, cudaEventDisableTiming)) != cudaSuccess)
        rc = fail("slow stream set-up", e);
    for (int r = 0; r < ring_blocks && rc == TG_OK; ++r) {
        cudaEvent_t l = nullptr, f = nullptr;
        if ((e = cudaEventCreateWithFlags(&l, cudaEventDisableTiming)) != cudaSuccess ||
            (e = cudaEventCreateWithFlags(&f, cudaEventDisableTiming)) != cudaSuccess)
            rc = fail("cudaEventCreateWithFlags", e);
        if (l) s->landed.push_back(l);
        if (f) s->freed.push_back(f);
    }
    cudaSetDevice(prev);
    if (rc != TG_OK) return rc;
    *out = hold.release();
    return TG_OK;
}

}  // namespace

extern "C" int tg_slow_stream_create(const tg_shape *shape, const int32_t *kv_len, const int32_t *fast_len,
                                     const int32_t *group_of_head, const int64_t *group_off, int32_t n_groups,
                                     const int32_t *slow_page_table, const int64_t *slow_head_off,
                                     int64_t slow_table_len, int32_t block_pages, int32_t ring_blocks,
                                     const tg_plan_opts *opts, tg_slow_stream **out) {
    return no_throw([&] {
        return slow_stream_create(shape, kv_len, fast_len, group_of_head, group_off, n_groups, slow_page_table,
                                  slow_head_off, slow_table_len, block_pages, ring_blocks, opts, out);
    });
}

extern "C" void tg_slow_stream_destroy(tg_slow_stream *s) {
    if (!s) return;
    int prev = 0;
    cudaGetDevice(&prev);
    if (!s->host_only) {
        cudaSetDevice(s->device);
        if (s->copy) cudaStreamSynchronize(s->copy);
    }
    release(s);
    cudaSetDevice(prev);
}

extern "C" int tg_slow_stream_blocks(const tg_slow_stream *s, int64_t *first_page, int32_t *pages,
                                     int32_t *tokens) {
    if (!s) return TG_EINVAL;
    const int64_t BH = static_cast<int64_t>(s->shape.B) * s->shape.Hkv;
    const size_t J = s->blk_first.size();
    if (first_page) std::copy(s->blk_first.begin(), s->blk_first.end(), first_page);
    if (pages) std::copy(s->blk_pages.begin(), s->blk_pages.end(), pages);
    if (tokens) std::copy(s->blk_len.begin(), s->blk_len.begin() + static_cast<int64_t>(J) * BH, tokens);
    return static_cast<int>(J);
}

extern "C" int tg_slow_stream_status(tg_slow_stream *s, tg_stream stream) {
    if (!s || s->host_only) return TG_EINVAL;
    int worst = tg_plan_status(s->fast, stream);
    for (tg_plan *p : s->blk) {
        const int rc = tg_plan_status(p, stream);
        if (worst == TG_OK) worst = rc;
    }
    return worst;
}

extern "C" int tg_tiered_decode_streamed(tg_slow_stream *s, const void *q, const int8_t *k_q8_host,
                                         const int8_t *v_q8_host, const float *k_scale_host,
                                         const float *v_scale_host, const void *k_fast, const void *v_fast,
                                         const int32_t *fast_page_table, const int64_t *fast_head_off,
                                         const int32_t *group_of_head, float scale, void *out, float *lse,
                                         tg_stream stream_) {
    if (!s || s->host_only || !q || !out || !lse) return TG_EINVAL;
    const int64_t J = static_cast<int64_t>(s->blk.size());
    if (J > 0 && (!k_q8_host || !v_q8_host || !k_scale_host || !v_scale_host || !pinned(k_q8_host) ||
                  !pinned(v_q8_host) || !pinned(k_scale_host) || !pinned(v_scale_host)))
        return TG_EINVAL;
    int cur = 0;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return fail("cudaGetDevice", e);
    if (cur != s->device) return TG_EINVAL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    const tg_shape &S = s->shape;
    const int64_t BH = static_cast<int64_t>(S.B) * S.Hkv;
    const size_t D = static_cast<size_t>(S.D);
    const int64_t rows = static_cast<int64_t>(S.B) * S.Hq;
    const size_t R = static_cast<size_t>(s->row_bytes);
    const size_t slot_codes = static_cast<size_t>(s->block_pages) * 16 * R;
    const size_t slot_scales = static_cast<size_t>(s->block_pages) * 16;
    // Copies never start before the work already queued on `stream` (this call's inputs).
    if ((e = cudaEventRecord(s->start, stream)) != cudaSuccess || (e = cudaStreamWaitEvent(s->copy, s->start, 0)) != cudaSuccess)
        return fail("slow stream: start", e);
    auto fast_decode = [&]() {
        return tg_ragged_paged_decode(s->fast, q, k_fast, v_fast, fast_page_table, fast_head_off, s->d_fast_len,
                                      group_of_head, scale, s->part_o, s->part_lse, stream_);
    };
    int rc = TG_OK;
    if (J == 0) rc = fast_decode();
    for (int64_t j = 0; j < J && rc == TG_OK; ++j) {
        const int r = static_cast<int>(j % s->ring);
        const size_t pages = static_cast<size_t>(s->blk_pages[j]);
        const size_t first = static_cast<size_t>(s->blk_first[j]);
        int8_t *rk = s->ring_k + r * slot_codes, *rv = s->ring_v + r * slot_codes;
        float *rks = s->ring_ks + r * slot_scales, *rvs = s->ring_vs + r * slot_scales;
        if ((e = cudaStreamWaitEvent(s->copy, s->freed[r], 0)) != cudaSuccess ||
            (e = cudaMemcpyAsync(rk, k_q8_host + first * 16 * R, pages * 16 * R, cudaMemcpyHostToDevice, s->copy)) != cudaSuccess ||
            (e = cudaMemcpyAsync(rv, v_q8_host + first * 16 * R, pages * 16 * R, cudaMemcpyHostToDevice, s->copy)) != cudaSuccess ||
            (e = cudaMemcpyAsync(rks, k_scale_host + first * 16, pages * 16 * 4, cudaMemcpyHostToDevice, s->copy)) != cudaSuccess ||
            (e = cudaMemcpyAsync(rvs, v_scale_host + first * 16, pages * 16 * 4, cudaMemcpyHostToDevice, s->copy)) != cudaSuccess ||
            (e = cudaEventRecord(s->landed[r], s->copy)) != cudaSuccess)
            return fail("slow stream: block copy", e);
        if (j == 0 && (rc = fast_decode()) != TG_OK) break;  // overlaps the first copy
        if ((e = cudaStreamWaitEvent(stream, s->landed[r], 0)) != cudaSuccess) return fail("slow stream: wait", e);
        rc = tg_tiered_decode(s->blk[j], q, rk, rv, rks, rvs, s->d_table + s->blk_table_base[j], s->d_off + j * BH,
                              nullptr, nullptr,
                              nullptr, nullptr, s->d_len + j * BH, s->d_zero, scale,
                              s->part_o + static_cast<size_t>(1 + j) * rows * D,
                              s->part_lse + static_cast<size_t>(1 + j) * rows, stream_);
        if (rc != TG_OK) break;
        if ((e = cudaEventRecord(s->freed[r], stream)) != cudaSuccess) return fail("slow stream: freed", e);
    }
    if (rc != TG_OK) return rc;
    const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
    if (S.D == 128)
        stream_merge_kernel<128><<<grid, 256, 0, stream>>>(static_cast<int32_t>(1 + J), rows, s->part_o, s->part_lse,
                                                           static_cast<__nv_bfloat16 *>(out), lse);
    else
        stream_merge_kernel<64><<<grid, 256, 0, stream>>>(static_cast<int32_t>(1 + J), rows, s->part_o, s->part_lse,
                                                          static_cast<__nv_bfloat16 *>(out), lse);
    if ((e = cudaGetLastError()) != cudaSuccess) return fail("stream_merge_kernel", e);
    return TG_OK;
}
