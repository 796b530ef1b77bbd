// CUDA side of libtg (sm_100a): split-K ragged / tiered paged decode, the log-sum-exp merge,
// the INT8 slow-tier quantiser, plan device state and launchers.
//
// Decode kernel design (one layer, one step):
//   * Persistent CTAs of kPairs (producer warp, consumer warp) pairs; each pair is one worker
//     of the static plan and walks its items (page ranges of one (sequence, KV head) row).
//   * The producer warp reads the page ids through the table and streams each page's K and V
//     into a per-pair ring of shared-memory stages with the Tensor Memory Accelerator
//     (2-D tiled loads, 128-byte swizzle, mbarrier transaction counts; no clusters, no
//     multicast). The first page of an item also brings the item's G query rows; INT8 pages
//     also bring their per-token fp32 scales.
//   * The consumer warp computes S = K q^T for 16 tokens x (up to) 8 query heads with
//     mma.m16n8k16 (tokens on M, the GQA heads of the KV head on N), an online softmax in
//     the log2 domain, and O^T += V^T P^T with the head dimension on M. INT8 rows are
//     converted exactly to fp16 in registers; their scales multiply the score (K) and the
//     probability (V) in fp32.
//   * Items that cover a whole head write bf16 out + fp32 lse; split heads write normalised
//     fp32 partials that the merge kernel combines by log-sum-exp in split order.
//   * Every wait is bounded (globaltimer); every page id and table row is range-checked
//     before a copy is issued. Faults turn into bits of the plan's error word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "tg_internal.h"

namespace tg {

// ------------------------------------------------------------------------------------------
// Error reporting
// ------------------------------------------------------------------------------------------
static thread_local char g_cuda_msg[256] = "";

void set_cuda_error(const char *what, int code) {
    std::snprintf(g_cuda_msg, sizeof(g_cuda_msg), "%s: %s (%d)", what,
                  cudaGetErrorString(static_cast<cudaError_t>(code)), code);
}

#define TG_CUDA_TRY(expr)                                   \
    do {                                                    \
        cudaError_t e_ = (expr);                            \
        if (e_ != cudaSuccess) {                            \
            set_cuda_error(#expr, static_cast<int>(e_));    \
            return TG_ECUDA;                                \
        }                                                   \
    } while (0)

// ------------------------------------------------------------------------------------------
// Device helpers (inline PTX)
// ------------------------------------------------------------------------------------------
namespace dev {

constexpr uint64_t kDrainNs = 200000000ull;  // bound of the drain after a timeout: 0.2 s

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test: has the phase of the given parity completed?
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase of the given parity; false after `limit` ns.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer();
    while (!mbar_try_wait(bar, parity))
        if (global_timer() - t0 > limit) return false;
    return true;
}

// 2-D tiled TMA load into this CTA's shared memory, completing on an mbarrier.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, int32_t x, int32_t y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ uint32_t movm_t(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Unsigned A (INT4 codes widened to offset-binary bytes 0..15) against signed B.
__device__ __forceinline__ void mma_u8s8(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_s8(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Hardware base-2 exponential and logarithm (PTX ex2.approx / lg2.approx).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float f16_lo(uint32_t v) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(v & 0xFFFFu)));
}
__device__ __forceinline__ float f16_hi(uint32_t v) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(v >> 16)));
}

// One ldmatrix.trans register of INT8 V codes, bytes (x[t][d], x[t][d+1], x[t+1][d], x[t+1][d+1]),
// -> two fp16x2 registers (x[t][d], x[t+1][d]) and (x[t][d+1], x[t+1][d+1]) holding x + 1152,
// exactly: bias each byte to x + 128 and place it in the low mantissa byte of fp16 1024 (0x6400).
// The constant 1152 is not subtracted here: the P V product carries 1152 sum(p') per head, which
// the item's end removes once (kV8Offset).
__device__ __forceinline__ void i8pair_to_f16(uint32_t v, uint32_t &lo, uint32_t &hi) {
    const uint32_t u = v ^ 0x80808080u;
    asm("prmt.b32 %0, %1, %2, 0x4240;" : "=r"(lo) : "r"(u), "r"(0x64646464u));
    asm("prmt.b32 %0, %1, %2, 0x4341;" : "=r"(hi) : "r"(u), "r"(0x64646464u));
}
constexpr float kV8Offset = 1152.f;

// One ldmatrix.trans register of INT4 V (offset-binary nibbles u = x + 8; bits 0-7 token t byte
// b, 8-15 token t byte b+1, 16-23 token t+1 byte b, 24-31 token t+1 byte b+1) -> fp16x2 (t, t+1)
// of its four d, exactly and with the offsets left in: `lo` takes the low nibbles of bytes b
// (shift 0) or b+1 (shift 8) as 1024 + u = x + 1032; `hi` the high nibbles as 1024 + 16 u =
// 16 x + 1152, i.e. 16 (x + 72). The item's end scales the high-nibble tiles by 1/16 and removes
// 1032 or 72 times sum(p') per head.
__device__ __forceinline__ uint32_t nib_lo_f16(uint32_t v) { return (v & 0x000F000Fu) | 0x64006400u; }
__device__ __forceinline__ uint32_t nib_hi_f16(uint32_t v) { return (v & 0x00F000F0u) | 0x64006400u; }
constexpr float kV4LoOffset = 1032.f, kV4HiOffset = 72.f;

// Byte offset of 16-byte chunk `chunk` of row `row` in a box of 64-byte rows written by TMA
// with 64-byte swizzle (chunk bits XOR address bits 7-8; the box base is 512-byte aligned).
__device__ __forceinline__ uint32_t swz64(uint32_t row, uint32_t chunk) {
    return row * 64u + (((chunk ^ (row >> 1)) & 3u) << 4);
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a box of 128-byte rows written by TMA
// with 128-byte swizzle (the box base is 1024-byte aligned).
__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {
    return row * 128u + (((chunk ^ row) & 7u) << 4);
}

}  // namespace dev
// ------------------------------------------------------------------------------------------
// Kernel arguments
// ------------------------------------------------------------------------------------------
struct DecodeArgs {
    const Item *items;
    const int32_t *worker_off;
    int32_t n_workers;
    int32_t B, Hq, Hkv, G;
    int32_t stages, stage_bytes;
    float scale_log2;                // softmax scale * log2(e)
    const __nv_bfloat16 *q;          // [B][Hq][D]
    const int32_t *table;            // bf16 (fast) tier table
    const int64_t *head_off;         // [B*Hkv]
    const int32_t *group_of_head;    // [Hkv]; null = bound rows by the whole table
    const int64_t *group_off;        // [n_groups + 1] (device copy in the plan)
    int32_t n_groups;
    const int32_t *slow_table;       // INT8 tier table (tiered)
    const int64_t *slow_off;         // [B*Hkv] (tiered)
    int64_t slow_table_len;
    const float *k_scale, *v_scale;  // [num_slow_pages][16] (tiered)
    const int32_t *kv_len_dev;       // [B*Hkv]
    const int32_t *fast_len_dev;     // [B*Hkv] (tiered) or null
    int64_t num_pages, num_slow_pages;
    __nv_bfloat16 *out;              // [B][Hq][D]
    float *out_f32;                  // [B][Hq][D] instead of out (plans with out_f32), else null
    float *lse;                      // [B][Hq]
    float *part_o;                   // [n_partials][G][D]
    float *part_lse;                 // [n_partials][G]
    const int32_t *empties;          // heads with no tokens
    int32_t n_empty;
    int32_t dyn_first, n_dyn;        // dynamic items: items[dyn_first .. dyn_first + n_dyn)
    uint32_t *dyn_next;              // [0] next dynamic item, [1] producers done (zero between calls)
    int32_t early_prologue;          // read plan/table metadata before the predecessor finishes
    uint64_t wait_ns;                // bound of any single wait
    int32_t withhold;                // testing: worker 0 never signals its page number withhold
    uint32_t *err;
    uint64_t *trace;                 // worker timeline (n_workers x kTraceWords) or null
    float *token_scores;             // bf16 kernel: per-token scores [table_len*16][G], or null
    int32_t late_wait;               // wait for the preceding grid only before exiting (cascade
                                     // plans: that grid is the cascade kernel, independent work)
    int32_t capacity;                // tiered: planned lengths are capacities; tier token counts
                                     // come from the device lengths of each call
};

// Per-stage header written by the producer before it arrives on the stage's full barrier.
struct alignas(16) StageHdr {
    int32_t valid;  // valid tokens in this page (0 when the page was skipped)
    int32_t flags;  // kHdr* bits
    int32_t bh;
    int32_t slot;
    int64_t tpos;   // table position of the page (head row offset + page index in the row)
    int64_t pad;
};
constexpr int32_t kHdrSlow = 1, kHdrFirst = 2, kHdrLast = 4, kHdrStop = 8, kHdrPair = 16;
constexpr int32_t kNoLoad = -2;  // page id placeholder of a row that failed its bounds check

// Shared-memory stage layout (offsets within a stage; D = 128 shown, D = 64 halves the bf16
// regions): K bf16 [0, KB) as D/64 boxes of 16 rows x 128 B; V bf16 [KB, 2KB); q [2KB, +QB).
// INT8 pages reuse it: K codes [0, 2048), K scales [2048, 2112), V scales [2112, 2176),
// V codes [KB, KB + 2048). INT4 pages: packed K [KB + 2048, KB + 3072), packed V
// [KB + 3072, KB + 4096) (16 rows x 64 B each, 64-byte swizzle), scales as INT8.
template <int D>
struct Layout {
    static constexpr int KB = 16 * D * 2;
    static constexpr int kI8 = 16 * D;  // one INT8 page of one tensor
    static constexpr int kI4 = 8 * D;   // one INT4 page of one tensor
    static constexpr int kKScale = 2048, kVScale = 2112;
    static constexpr int kK4 = KB + kI8, kV4 = KB + kI8 + kI4;
};

// Online-softmax state of the two query heads (2t, 2t+1) a consumer lane accumulates.
struct PageState {
    float sq0, sq1;  // INT8 tier: s_q * scale * log2(e) / 254 of heads 2t, 2t+1
    int32_t k0, k1;  // INT4 tier: 8 (254 sum q1 + sum q2) of heads 2t, 2t+1 (offset-binary K)
    float m0, m1;    // running maxima, log2 units
    float le0, le1;  // sums of fp32 probabilities (for the lse)
    float lr0, lr1;  // sums of the probabilities multiplied into V
    float w0, w1;    // slow tiers: sums of the fp16 p' = p * v_scale that met the offset V codes
    __device__ __forceinline__ void reset() {
        m0 = m1 = -INFINITY;
        le0 = le1 = lr0 = lr1 = w0 = w1 = 0.f;
    }
};

// One consumer step over NP pages (1 or 2) of the same item: S = K q^T per page (16 tokens x
// 8 heads, tokens on M), one max reduction and rescale check for all NP pages, then O^T +=
// V^T P^T per page. With NP = 2 the two pages' instruction streams interleave (independent
// chains). SLOW: INT8 pages (K codes on the s8 tensor path against two int8 digits of q, V codes
// widened to fp16 in registers, per-token scales); with SB = 4 the pages hold INT4 codes (byte
// i of a row: d = i low nibble, d = i + D/2 high nibble, offset-binary), and off8[0..1] are the
// ldmatrix offsets of the two 32-byte halves of the 64-byte rows.
template <int D, int NP, bool SLOW, int SB = 8>
__device__ __forceinline__ void consume_pages(const uint32_t (&sa)[NP], const int (&valid)[NP],
                                              const uint32_t (&qf)[D / 16][2],
                                              float (&o)[D / 16][4], PageState &ps,
                                              const uint32_t (&offK)[D / 16],
                                              const uint32_t (&offV)[D / 16],
                                              const uint32_t (&off8)[D / 32], float scale_log2,
                                              int lane, float *ts = nullptr, int64_t tpos = 0,
                                              int32_t G = 0) {
    using L = Layout<D>;
    constexpr int KS = D / 16;
    constexpr unsigned FULL = 0xffffffffu;
    const int g = lane >> 2, t = lane & 3;
    float s[NP][4];
    float ks[NP][2], vs[NP][2];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        s[p][0] = s[p][1] = s[p][2] = s[p][3] = 0.f;
        ks[p][0] = ks[p][1] = vs[p][0] = vs[p][1] = 1.f;
    }
    if (!SLOW) {
#pragma unroll
        for (int j = 0; j < KS; ++j) {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                uint32_t a0, a1, a2, a3;
                dev::ldsm_x4(sa[p] + offK[j], a0, a1, a2, a3);
                dev::mma_bf16(s[p], a0, a1, a2, a3, qf[j][0], qf[j][1]);
            }
        }
    } else if (SB == 4) {
        // INT4 K: one ldmatrix of a 32-byte half gives, per register, four bytes of one token;
        // their low nibbles are the u8 A fragment of d chunk jj and their high nibbles that of
        // chunk jj + 2 (d + 64). S = s_q (K.q1 + K.q2 / 254) with K = u - 8: the 8 (254 sum q1
        // + sum q2) of the offset is subtracted in int32 (ps.k0 / ps.k1).
        int32_t s1[NP][4], s2[NP][4];
#pragma unroll
        for (int p = 0; p < NP; ++p) s1[p][0] = s1[p][1] = s1[p][2] = s1[p][3] = s2[p][0] = s2[p][1] = s2[p][2] = s2[p][3] = 0;
#pragma unroll
        for (int jj = 0; jj < D / 64; ++jj) {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                uint32_t r0, r1, r2, r3;
                dev::ldsm_x4(sa[p] + L::kK4 + off8[jj], r0, r1, r2, r3);
                const uint32_t m = 0x0F0F0F0Fu;
                dev::mma_u8s8(s1[p], r0 & m, r1 & m, r2 & m, r3 & m, qf[jj][0], qf[jj][1]);
                dev::mma_u8s8(s2[p], r0 & m, r1 & m, r2 & m, r3 & m, qf[KS / 2 + jj][0], qf[KS / 2 + jj][1]);
                dev::mma_u8s8(s1[p], (r0 >> 4) & m, (r1 >> 4) & m, (r2 >> 4) & m, (r3 >> 4) & m,
                              qf[jj + D / 64][0], qf[jj + D / 64][1]);
                dev::mma_u8s8(s2[p], (r0 >> 4) & m, (r1 >> 4) & m, (r2 >> 4) & m, (r3 >> 4) & m,
                              qf[KS / 2 + jj + D / 64][0], qf[KS / 2 + jj + D / 64][1]);
            }
        }
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            s[p][0] = static_cast<float>(s1[p][0] * 254 + s2[p][0] - ps.k0);
            s[p][1] = static_cast<float>(s1[p][1] * 254 + s2[p][1] - ps.k1);
            s[p][2] = static_cast<float>(s1[p][2] * 254 + s2[p][2] - ps.k0);
            s[p][3] = static_cast<float>(s1[p][3] * 254 + s2[p][3] - ps.k1);
        }
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            float k0, k1, v0, v1;
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(k0) : "r"(sa[p] + L::kKScale + 4 * g));
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(k1) : "r"(sa[p] + L::kKScale + 4 * (g + 8)));
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v0) : "r"(sa[p] + L::kVScale + 4 * g));
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v1) : "r"(sa[p] + L::kVScale + 4 * (g + 8)));
            ks[p][0] = k0;
            ks[p][1] = k1;
            vs[p][0] = v0;
            vs[p][1] = v1;
        }
    } else {
        // INT8 codes straight into the integer tensor-core path: K (tokens x 32 d, as stored)
        // times the two int8 digits of q; S = s_q * (K.q1 + K.q2 / 254), exact in int32.
        int32_t s1[NP][4], s2[NP][4];
#pragma unroll
        for (int p = 0; p < NP; ++p) s1[p][0] = s1[p][1] = s1[p][2] = s1[p][3] = s2[p][0] = s2[p][1] = s2[p][2] = s2[p][3] = 0;
#pragma unroll
        for (int jj = 0; jj < KS / 2; ++jj) {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                uint32_t r0, r1, r2, r3;
                dev::ldsm_x4(sa[p] + off8[jj], r0, r1, r2, r3);
                dev::mma_s8(s1[p], r0, r1, r2, r3, qf[jj][0], qf[jj][1]);
                dev::mma_s8(s2[p], r0, r1, r2, r3, qf[KS / 2 + jj][0], qf[KS / 2 + jj][1]);
            }
        }
        // 254 s1 + s2 is exact in int32 (|s1| < 2^21); ps.sq* carries s_q * scale * log2(e) / 254.
#pragma unroll
        for (int p = 0; p < NP; ++p) {
#pragma unroll
            for (int c = 0; c < 4; ++c) s[p][c] = static_cast<float>(s1[p][c] * 254 + s2[p][c]);
        }
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            float k0, k1, v0, v1;
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(k0) : "r"(sa[p] + L::kKScale + 4 * g));
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(k1) : "r"(sa[p] + L::kKScale + 4 * (g + 8)));
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v0) : "r"(sa[p] + L::kVScale + 4 * g));
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v1) : "r"(sa[p] + L::kVScale + 4 * (g + 8)));
            ks[p][0] = k0;
            ks[p][1] = k1;
            vs[p][0] = v0;
            vs[p][1] = v1;
        }
    }
    // s[p][0]: token g head 2t; s[p][1]: token g head 2t+1; s[p][2]/s[p][3]: token g+8.
    float x[NP][4];
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const bool v0 = g < valid[p], v1 = g + 8 < valid[p];
        const float f0 = SLOW ? ks[p][0] * ps.sq0 : scale_log2, f1 = SLOW ? ks[p][0] * ps.sq1 : scale_log2;
        const float f2 = SLOW ? ks[p][1] * ps.sq0 : scale_log2, f3 = SLOW ? ks[p][1] * ps.sq1 : scale_log2;
        x[p][0] = v0 ? s[p][0] * f0 : -INFINITY;
        x[p][1] = v0 ? s[p][1] * f1 : -INFINITY;
        x[p][2] = v1 ? s[p][2] * f2 : -INFINITY;
        x[p][3] = v1 ? s[p][3] * f3 : -INFINITY;
        mx0 = fmaxf(mx0, fmaxf(x[p][0], x[p][2]));
        mx1 = fmaxf(mx1, fmaxf(x[p][1], x[p][3]));
    }
    if (!SLOW && ts != nullptr) {
        // Per-token scores s = x * ln 2 of the valid tokens, entry (tpos * 16 + token) * G + head.
        constexpr float kLn2f = 0.69314718055994530942f;
        const int n0 = 2 * t, n1 = 2 * t + 1;
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            float *e0 = ts + ((tpos + p) * 16 + g) * G;
            float *e1 = e0 + 8 * G;
            if (g < valid[p]) {
                if (n0 < G) e0[n0] = x[p][0] * kLn2f;
                if (n1 < G) e0[n1] = x[p][1] * kLn2f;
            }
            if (g + 8 < valid[p]) {
                if (n0 < G) e1[n0] = x[p][2] * kLn2f;
                if (n1 < G) e1[n1] = x[p][3] * kLn2f;
            }
        }
    }
    // Lazy rescale: the running max moves only when a tile exceeds it by more than the
    // threshold (2^8 for bf16 probabilities; exact for the fp16 INT8 path). A lane's own
    // maxima decide whether any head's tile maximum does (the running max is the same across
    // a head's lanes), so the cross-lane reduction runs only when it will be used.
    const float thr = SLOW ? 0.f : 8.f;
    if (__any_sync(FULL, mx0 > ps.m0 + thr || mx1 > ps.m1 + thr)) {
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, off));
        }
        const bool up0 = mx0 > ps.m0 + thr, up1 = mx1 > ps.m1 + thr;
        const float n0 = up0 ? mx0 : ps.m0, n1 = up1 ? mx1 : ps.m1;
        const float c0 = (ps.m0 == -INFINITY) ? 0.f : dev::ex2(ps.m0 - n0);
        const float c1 = (ps.m1 == -INFINITY) ? 0.f : dev::ex2(ps.m1 - n1);
#pragma unroll
        for (int i = 0; i < KS; ++i) {
            o[i][0] *= c0;
            o[i][1] *= c1;
            o[i][2] *= c0;
            o[i][3] *= c1;
        }
        ps.le0 *= c0;
        ps.le1 *= c1;
        ps.lr0 *= c0;
        ps.lr1 *= c1;
        if (SLOW) {
            ps.w0 *= c0;
            ps.w1 *= c1;
        }
        ps.m0 = n0;
        ps.m1 = n1;
    }
    float pv[NP][4];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        pv[p][0] = x[p][0] == -INFINITY ? 0.f : dev::ex2(x[p][0] - ps.m0);
        pv[p][1] = x[p][1] == -INFINITY ? 0.f : dev::ex2(x[p][1] - ps.m1);
        pv[p][2] = x[p][2] == -INFINITY ? 0.f : dev::ex2(x[p][2] - ps.m0);
        pv[p][3] = x[p][3] == -INFINITY ? 0.f : dev::ex2(x[p][3] - ps.m1);
        ps.le0 += pv[p][0] + pv[p][2];
        ps.le1 += pv[p][1] + pv[p][3];
    }
    if (!SLOW) {
        uint32_t b0[NP], b1[NP], mk01[NP], mk23[NP];
        bool tail[NP];
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            const uint32_t r0 = dev::pack_bf16(pv[p][0], pv[p][1]), r1 = dev::pack_bf16(pv[p][2], pv[p][3]);
            ps.lr0 += dev::bf16_lo(r0) + dev::bf16_lo(r1);
            ps.lr1 += dev::bf16_hi(r0) + dev::bf16_hi(r1);
            b0[p] = dev::movm_t(r0);
            b1[p] = dev::movm_t(r1);
            // token masks of this thread's A-fragment halves (tokens 2t, 2t+1 | 2t+8, 2t+9)
            mk01[p] = (2 * t < valid[p] ? 0xFFFFu : 0u) | (2 * t + 1 < valid[p] ? 0xFFFF0000u : 0u);
            mk23[p] = (2 * t + 8 < valid[p] ? 0xFFFFu : 0u) | (2 * t + 9 < valid[p] ? 0xFFFF0000u : 0u);
            tail[p] = valid[p] < 16;
        }
#pragma unroll
        for (int i = 0; i < KS; ++i) {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                uint32_t a0, a1, a2, a3;
                dev::ldsm_x4_t(sa[p] + offV[i], a0, a1, a2, a3);
                if (tail[p]) {
                    a0 &= mk01[p];
                    a1 &= mk01[p];
                    a2 &= mk23[p];
                    a3 &= mk23[p];
                }
                dev::mma_bf16(o[i], a0, a1, a2, a3, b0[p], b1[p]);
            }
        }
    } else {
        uint32_t b0[NP], b1[NP];
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            // p' = p * v_scale (fp32) -> fp16; the normaliser keeps the unscaled p.
            ps.lr0 += pv[p][0] + pv[p][2];
            ps.lr1 += pv[p][1] + pv[p][3];
            const bool v0 = g < valid[p], v1 = g + 8 < valid[p];
            const float q0 = v0 ? pv[p][0] * vs[p][0] : 0.f, q1 = v0 ? pv[p][1] * vs[p][0] : 0.f;
            const float q2 = v1 ? pv[p][2] * vs[p][1] : 0.f, q3 = v1 ? pv[p][3] * vs[p][1] : 0.f;
            const uint32_t h01 = dev::pack_f16(q0, q1), h23 = dev::pack_f16(q2, q3);
            ps.w0 += dev::f16_lo(h01) + dev::f16_lo(h23);
            ps.w1 += dev::f16_hi(h01) + dev::f16_hi(h23);
            b0[p] = dev::movm_t(h01);
            b1[p] = dev::movm_t(h23);
        }
        if (SB == 4) {
            // INT4 V: ldmatrix.trans of a 32-byte half jj (chunks 2jj, 2jj+1): r0 / r1 tokens
            // (2t, 2t+1) / (8+2t, 9+2t) at bytes 32jj + 2g, +1, r2 / r3 the same 16 bytes on.
            // Low nibbles: d tiles 2jj and 2jj+1; high nibbles: the tiles D/32 further (d + D/2);
            // row g -> d 16i + 2g (byte b), row g+8 -> d + 1 (byte b+1), as on the INT8 path.
#pragma unroll
            for (int jj = 0; jj < D / 64; ++jj) {
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    uint32_t r0, r1, r2, r3;
                    dev::ldsm_x4_t(sa[p] + L::kV4 + off8[jj], r0, r1, r2, r3);
                    dev::mma_f16(o[2 * jj], dev::nib_lo_f16(r0), dev::nib_lo_f16(r0 >> 8), dev::nib_lo_f16(r1),
                                 dev::nib_lo_f16(r1 >> 8), b0[p], b1[p]);
                    dev::mma_f16(o[2 * jj + D / 32], dev::nib_hi_f16(r0), dev::nib_hi_f16(r0 >> 8),
                                 dev::nib_hi_f16(r1), dev::nib_hi_f16(r1 >> 8), b0[p], b1[p]);
                    dev::mma_f16(o[2 * jj + 1], dev::nib_lo_f16(r2), dev::nib_lo_f16(r2 >> 8), dev::nib_lo_f16(r3),
                                 dev::nib_lo_f16(r3 >> 8), b0[p], b1[p]);
                    dev::mma_f16(o[2 * jj + 1 + D / 32], dev::nib_hi_f16(r2), dev::nib_hi_f16(r2 >> 8),
                                 dev::nib_hi_f16(r3), dev::nib_hi_f16(r3 >> 8), b0[p], b1[p]);
                }
            }
        } else {
#pragma unroll
        for (int ii = 0; ii < KS / 2; ++ii) {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                uint32_t r0, r1, r2, r3;
                dev::ldsm_x4_t(sa[p] + L::KB + off8[ii], r0, r1, r2, r3);
                // r0/r1: tokens (2t, 2t+1) / (8+2t, 9+2t) at d = 32ii + 2g, +1 (chunk 2ii);
                // r2/r3: the same for chunk 2ii+1. Tile i rows: g -> d 16i + 2g, g+8 -> +1.
                uint32_t a0, a1, a2, a3;
                dev::i8pair_to_f16(r0, a0, a1);
                dev::i8pair_to_f16(r1, a2, a3);
                dev::mma_f16(o[2 * ii], a0, a1, a2, a3, b0[p], b1[p]);
                dev::i8pair_to_f16(r2, a0, a1);
                dev::i8pair_to_f16(r3, a2, a3);
                dev::mma_f16(o[2 * ii + 1], a0, a1, a2, a3, b0[p], b1[p]);
            }
        }
        }
    }
}

// ------------------------------------------------------------------------------------------
// Decode kernel
// ------------------------------------------------------------------------------------------
constexpr int kIssueLanes = 8;  // most pages one producer batch issues (lane l: page k + l)

template <int D, bool TIERED, int NPAIRS, int SB = 8>
__global__ void __launch_bounds__(NPAIRS * 64, 1)
    decode_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_kq,
                  const __grid_constant__ CUtensorMap tm_vq) {
    using L = Layout<D>;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    // Warps [0, NPAIRS) consume, warps [NPAIRS, 2 NPAIRS) produce; pair p = warps p, NPAIRS + p.
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = warp % NPAIRS;
    const bool producer = warp >= NPAIRS;
    const int stages = a.stages;
    const int worker = blockIdx.x * NPAIRS + pair;

    unsigned char *ring = smem + static_cast<size_t>(pair) * stages * a.stage_bytes;
    StageHdr *hdr = reinterpret_cast<StageHdr *>(smem + static_cast<size_t>(NPAIRS) * stages * a.stage_bytes) +
                    pair * stages;
    uint64_t *bars = reinterpret_cast<uint64_t *>(
                         smem + static_cast<size_t>(NPAIRS) * stages * a.stage_bytes +
                         static_cast<size_t>(NPAIRS) * stages * sizeof(StageHdr)) +
                     static_cast<size_t>(pair) * stages * 2;
    volatile int32_t *ctl = reinterpret_cast<volatile int32_t *>(
                                smem + static_cast<size_t>(NPAIRS) * stages * a.stage_bytes +
                                static_cast<size_t>(NPAIRS) * stages * (sizeof(StageHdr) + 16)) +
                            pair * 2;  // [0] = pages issued, [1] = abort

    const uint32_t full0 = dev::smem_addr(bars), empty0 = dev::smem_addr(bars + stages);
    if (lane == 0 && !producer) {
        for (int s = 0; s < stages; ++s) {
            dev::mbar_init(full0 + 8 * s, 1);
            dev::mbar_init(empty0 + 8 * s, 1);
        }
        ctl[0] = 0;
        ctl[1] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    // Programmatic dependent launch: the kernel that follows in the stream may be scheduled
    // now (it waits for this grid before touching what this grid writes). This grid waits for
    // its predecessor here, or, with early_prologue, only the producers read the plan and the
    // tables first and wait just before their first copy (queries, K/V and every write come
    // after the wait).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!a.late_wait && (!a.early_prologue || !producer)) asm volatile("griddepcontrol.wait;" ::: "memory");

    // Heads with no retained token: out = 0, lse = -inf (consumer warps).
    if (a.n_empty > 0 && !producer) {
        const int64_t per = static_cast<int64_t>(a.G) * D;
        const int64_t total = static_cast<int64_t>(a.n_empty) * per;
        const int64_t nthr = static_cast<int64_t>(gridDim.x) * NPAIRS * 32;
        for (int64_t i = (static_cast<int64_t>(blockIdx.x) * NPAIRS + pair) * 32 + lane; i < total; i += nthr) {
            const int32_t bh = a.empties[i / per];
            const int32_t b = bh / a.Hkv, h = bh - b * a.Hkv;
            const int64_t r = i % per;
            const int64_t row = static_cast<int64_t>(b) * a.Hq + static_cast<int64_t>(h) * a.G + r / D;
            if (a.out_f32)
                a.out_f32[row * D + r % D] = 0.f;
            else
                a.out[row * D + r % D] = __float2bfloat16_rn(0.f);
            if (r % D == 0) a.lse[row] = -INFINITY;
        }
    }

    // Static items of this worker (none for pairs beyond the plan's workers), then dynamic
    // items taken from a shared ticket until they run out, then a stop marker.
    const int it0 = worker < a.n_workers ? a.worker_off[worker] : 0;
    const int it1 = worker < a.n_workers ? a.worker_off[worker + 1] : 0;
    uint64_t *trace = (a.trace && worker < a.n_workers) ? a.trace + static_cast<size_t>(worker) * kTraceWords : nullptr;
    if (trace && lane == 0 && !producer) {
        trace[0] = dev::global_timer();
        trace[6] = trace[7] = 0;
    }
    if (trace && lane == 0 && producer) trace[5] = 0;

    if (producer) {
        // ================================ producer warp ================================
        // Items are taken up to 32 at a time: lane j holds item j's metadata and its row
        // offset, checked against its (group) table; page ids are read 32 at a time, one
        // block ahead.
        uint32_t seq = 0;
        int pstage = 0;        // seq % stages
        uint32_t pphase = 0;   // (seq / stages) & 1
        bool aborted = false;
        bool waited = !a.early_prologue || a.late_wait;
        auto wait_predecessor = [&]() {
            if (!waited) {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                waited = true;
            }
        };
        auto run_items = [&](int c0, int nc) {
            Item mi{};
            int64_t mrow = 0;
            int32_t mok = 0;
            int32_t mtt = 0;  // tokens of the item's tier in its head (this call's)
            if (lane < nc) {
                mi = a.items[c0 + lane];
                const bool slow = TIERED && (mi.flags & kItemSlow);
                const int32_t h = mi.bh % a.Hkv;
                const int32_t row_pages = (mi.tier_tokens + 15) >> 4;
                int64_t lo = 0, hi;
                if (slow) {
                    mrow = a.slow_off[mi.bh];
                    hi = a.slow_table_len;
                } else {
                    mrow = a.head_off[mi.bh];
                    lo = a.group_off[0];
                    hi = a.group_off[a.n_groups];
                    if (a.group_of_head) {
                        const int32_t g = a.group_of_head[h];
                        if (g >= 0 && g < a.n_groups) {
                            lo = a.group_off[g];
                            hi = a.group_off[g + 1];
                        } else {
                            hi = lo - 1;  // invalid group: reject the row
                        }
                    }
                }
                mok = (mrow >= lo && mrow + row_pages <= hi) ? 1 : 0;
                if (!mok) atomicOr(a.err, kErrBadRow);
                mtt = mi.tier_tokens;
                bool plan_ok;
                if (TIERED && a.capacity) {
                    // the plan reserved mi.fast_len fast and mi.kv_len - mi.fast_len slow slots
                    const int32_t n = a.kv_len_dev[mi.bh], f = a.fast_len_dev[mi.bh];
                    plan_ok = f >= 0 && f <= n && f <= mi.fast_len && n - f <= mi.kv_len - mi.fast_len;
                    mtt = !plan_ok ? 0 : (slow ? n - f : f);
                } else {
                    plan_ok = a.kv_len_dev[mi.bh] == mi.kv_len;
                    if (TIERED) plan_ok = plan_ok && a.fast_len_dev[mi.bh] == mi.fast_len;
                }
                if (!plan_ok) atomicOr(a.err, kErrPlan);
            }
            // Page ids of block (item j, pages p0 .. p0+31): lane k gets page p0 + k. The value
            // is not inspected here, so the load stays in flight until the block is issued.
            auto ids_of = [&](int j, int32_t p0) -> int32_t {
                const int64_t row = __shfl_sync(FULL, mrow, j);
                const int32_t ok = __shfl_sync(FULL, mok, j);
                const int32_t pe = __shfl_sync(FULL, mi.page_end, j);
                const int32_t fl = __shfl_sync(FULL, mi.flags, j);
                const bool slow = TIERED && (fl & kItemSlow);
                int32_t pid = kNoLoad;
                if (ok && lane < pe - p0) pid = __ldg((slow ? a.slow_table : a.table) + row + p0 + lane);
                return pid;
            };
            auto next_block = [&](int j, int32_t p0, int &jn, int32_t &pn) {
                const int32_t pe = __shfl_sync(FULL, mi.page_end, j);
                if (p0 + 32 < pe) {
                    jn = j;
                    pn = p0 + 32;
                } else {
                    jn = j + 1;
                    pn = jn < nc ? __shfl_sync(FULL, mi.page_begin, jn) : 0;
                }
            };
            int j = 0;
            int32_t p0 = __shfl_sync(FULL, mi.page_begin, 0);
            int32_t ids = ids_of(0, p0);
            int jn;
            int32_t pn;
            next_block(j, p0, jn, pn);
            int32_t ids_n = jn < nc ? ids_of(jn, pn) : kNoLoad;
            while (j < nc) {
                const int32_t bh = __shfl_sync(FULL, mi.bh, j);
                const int64_t row_j = __shfl_sync(FULL, mrow, j);
                const int32_t pb = __shfl_sync(FULL, mi.page_begin, j);
                const int32_t pe = __shfl_sync(FULL, mi.page_end, j);
                const int32_t tt = __shfl_sync(FULL, mtt, j);
                const int32_t slot = __shfl_sync(FULL, mi.slot, j);
                const int32_t fl = __shfl_sync(FULL, mi.flags, j);
                const bool slow = TIERED && (fl & kItemSlow);
                const int32_t b = bh / a.Hkv, h = bh - b * a.Hkv;
                const int32_t cnt = min(32, pe - p0);
                // Pages are issued in batches: the first free stage is waited for, the stages
                // after it that the consumer has already released (it releases a page pair at
                // once) are tested without waiting, and lane l issues page k + l of the block
                // into stage pstage + l, so the copies of up to kIssueLanes pages are issued
                // side by side instead of one after another from one lane.
                for (int32_t k = 0; k < cnt;) {
                    wait_predecessor();
                    const bool ok = dev::mbar_wait(empty0 + 8 * pstage, pphase ^ 1u, a.wait_ns);
                    if (!ok || ctl[1]) {
                        if (lane == 0) {
                            atomicOr(a.err, kErrTimeout);
                            ctl[1] = 1;
                        }
                        aborted = true;
                        return;
                    }
                    const int nmax = min(cnt - k, min(stages, kIssueLanes));
                    int stage = pstage + lane;
                    uint32_t phase = pphase;
                    if (stage >= stages) {
                        stage -= stages;
                        phase ^= 1u;
                    }
                    const bool is_free = lane == 0 ||
                                         (lane < nmax && dev::mbar_test(empty0 + 8 * stage, phase ^ 1u));
                    const uint32_t freed = __ballot_sync(FULL, is_free);
                    const int n = __ffs(~freed) - 1;  // released stages from pstage on, <= nmax
                    int32_t page_id = __shfl_sync(FULL, ids, (k + lane) & 31);
                    if (lane < n) {
                        const int32_t pg = p0 + k + lane;
                        const uint32_t sq = seq + static_cast<uint32_t>(lane);
                        const int32_t vtok = max(0, min(16, tt - pg * 16));
                        if (vtok == 0) {
                            page_id = kNoLoad;  // a reserved page holding no token yet
                        } else if (page_id != kNoLoad &&
                                   (page_id < 0 || page_id >= (slow ? a.num_slow_pages : a.num_pages))) {
                            atomicOr(a.err, kErrBadPage);
                            page_id = kNoLoad;
                        }
                        const bool first = pg == pb;
                        const bool last = pg == pe - 1;
                        // pages (pb, pb+1), (pb+2, pb+3), ... of an item are consumed together
                        const bool pair = ((pg - pb) & 1) == 0 && pg + 1 < pe;
                        StageHdr hd;
                        hd.valid = page_id >= 0 ? vtok : 0;
                        hd.flags = (slow ? kHdrSlow : 0) | (first ? kHdrFirst : 0) |
                                   (last ? kHdrLast : 0) | (pair ? kHdrPair : 0);
                        hd.bh = bh;
                        hd.slot = slot;
                        hd.tpos = row_j + pg;
                        hd.pad = 0;
                        hdr[stage] = hd;
                        const uint32_t st = dev::smem_addr(ring + static_cast<size_t>(stage) * a.stage_bytes);
                        const uint32_t fb = full0 + 8 * stage;
                        const uint32_t qbytes = static_cast<uint32_t>(a.G * D * 2);
                        uint32_t bytes = first ? qbytes : 0u;
                        if (page_id >= 0) bytes += slow ? 2u * ((SB == 4 ? L::kI4 : L::kI8) + 64u) : 2u * L::KB;
                        if (a.withhold && worker == 0 && sq + 1 == static_cast<uint32_t>(a.withhold)) {
                            // testing: this stage is never signalled; the consumer's bounded
                            // wait runs out and the call reports a timeout
                        } else if (bytes == 0) {
                            dev::mbar_arrive(fb);
                        } else {
                            dev::mbar_arrive_expect_tx(fb, bytes);
                            if (first)
                                dev::bulk_load(st + 2 * L::KB,
                                               a.q + (static_cast<int64_t>(b) * a.Hq + static_cast<int64_t>(h) * a.G) * D,
                                               qbytes, fb);
                            if (page_id >= 0) {
                                const int32_t y = page_id * 16;
                                if (slow && SB == 4) {
                                    dev::tma_load_2d(st + L::kK4, &tm_kq, 0, y, fb);
                                    dev::tma_load_2d(st + L::kV4, &tm_vq, 0, y, fb);
                                    dev::bulk_load(st + L::kKScale, a.k_scale + static_cast<int64_t>(page_id) * 16, 64, fb);
                                    dev::bulk_load(st + L::kVScale, a.v_scale + static_cast<int64_t>(page_id) * 16, 64, fb);
                                } else if (slow) {
                                    dev::tma_load_2d(st, &tm_kq, 0, y, fb);
                                    dev::tma_load_2d(st + L::KB, &tm_vq, 0, y, fb);
                                    dev::bulk_load(st + L::kKScale, a.k_scale + static_cast<int64_t>(page_id) * 16, 64, fb);
                                    dev::bulk_load(st + L::kVScale, a.v_scale + static_cast<int64_t>(page_id) * 16, 64, fb);
                                } else {
#pragma unroll
                                    for (int bx = 0; bx < D / 64; ++bx) {
                                        dev::tma_load_2d(st + bx * 2048, &tm_k, bx * 64, y, fb);
                                        dev::tma_load_2d(st + L::KB + bx * 2048, &tm_v, bx * 64, y, fb);
                                    }
                                }
                            }
                        }
                        if (trace && sq == 0) trace[1] = dev::global_timer();
                    }
                    __syncwarp();
                    if (lane == 0) ctl[0] = static_cast<int32_t>(seq + static_cast<uint32_t>(n));
                    seq += static_cast<uint32_t>(n);
                    pstage += n;
                    if (pstage >= stages) {
                        pstage -= stages;
                        pphase ^= 1u;
                    }
                    k += n;
                }
                j = jn;
                p0 = pn;
                ids = ids_n;
                if (j < nc) {
                    next_block(j, p0, jn, pn);
                    ids_n = jn < nc ? ids_of(jn, pn) : kNoLoad;
                }
            }
        };
        for (int c0 = it0; c0 < it1 && !aborted; c0 += 32) run_items(c0, min(32, it1 - c0));
        wait_predecessor();
        while (!aborted && a.n_dyn > 0) {
            uint32_t idx = 0;
            if (lane == 0) idx = atomicAdd(a.dyn_next, 1u);
            idx = __shfl_sync(FULL, idx, 0);
            if (idx >= static_cast<uint32_t>(a.n_dyn)) break;
            run_items(a.dyn_first + static_cast<int>(idx), 1);
            if (trace && lane == 0) trace[5] += 1;
        }
        if (!aborted) {
            // Stop marker for the consumer.
            const int stage = pstage;
            const uint32_t phase = pphase;
            if (!dev::mbar_wait(empty0 + 8 * stage, phase ^ 1u, a.wait_ns) || ctl[1]) {
                if (lane == 0) {
                    atomicOr(a.err, kErrTimeout);
                    ctl[1] = 1;
                }
            } else if (lane == 0) {
                StageHdr hd;
                hd.valid = 0;
                hd.flags = kHdrStop;
                hd.bh = 0;
                hd.slot = -1;
                hd.tpos = 0;
                hd.pad = 0;
                hdr[stage] = hd;
                dev::mbar_arrive(full0 + 8 * stage);
                ctl[0] = static_cast<int32_t>(seq + 1);
            }
            // The last producer of the launch to finish resets the dynamic queue.
            if (lane == 0 && a.n_dyn > 0) {
                __threadfence();
                const uint32_t total = gridDim.x * NPAIRS;
                if (atomicAdd(a.dyn_next + 1, 1u) == total - 1) {
                    a.dyn_next[0] = 0;
                    a.dyn_next[1] = 0;
                }
            }
        }
        if (a.late_wait) asm volatile("griddepcontrol.wait;" ::: "memory");
        return;
    }

    // ================================ consumer warp ================================
    const int g = lane >> 2, t = lane & 3;
    // Per-lane ldmatrix row offsets within a stage (128-byte swizzled boxes), fixed for the
    // whole kernel: bf16 K per k-step, bf16 V per m-tile, INT8 K/V per pair of 16-byte chunks.
    constexpr int KSTEPS = D / 16;
    uint32_t offK[KSTEPS], offV[KSTEPS], off8[KSTEPS / 2];
    {
        const int lm = lane >> 3;
#pragma unroll
        for (int j = 0; j < KSTEPS; ++j) {
            const uint32_t rk = (lm & 1) * 8 + (lane & 7), ck = 2 * j + (lm >> 1);
            offK[j] = (ck >> 3) * 2048 + dev::swz(rk, ck & 7);
            const uint32_t rv = (lm >> 1) * 8 + (lane & 7), cv = 2 * j + (lm & 1);
            offV[j] = L::KB + (cv >> 3) * 2048 + dev::swz(rv, cv & 7);
        }
#pragma unroll
        for (int j = 0; j < KSTEPS / 2; ++j)
            off8[j] = SB == 4 ? dev::swz64((lm & 1) * 8 + (lane & 7), 2 * j + (lm >> 1))
                              : dev::swz((lm & 1) * 8 + (lane & 7), 2 * j + (lm >> 1));
    }
    uint32_t qf[KSTEPS][2];
    float o[KSTEPS][4];
    // running max (log2 units) and normalisers of heads 2t, 2t+1: le = sum of fp32 p (for
    // lse), lr = sum of the p actually multiplied into V (bf16-rounded on the bf16 path)
    PageState ps;
    bool item_slow = false;
    uint32_t seq = 0;
    int cstage = 0;
    uint32_t cphase = 0;
    auto advance = [&]() {
        ++seq;
        if (++cstage == stages) {
            cstage = 0;
            cphase ^= 1u;
        }
    };
    auto timed_out = [&]() {
        // Stop the producer and drain the copies it issued, then leave.
        if (lane == 0) {
            atomicOr(a.err, kErrTimeout);
            ctl[1] = 1;
        }
        __syncwarp();
        const uint32_t issued = static_cast<uint32_t>(ctl[0]);
        for (uint32_t s = seq; s < issued; ++s)
            dev::mbar_wait(full0 + 8 * (s % stages), (s / stages) & 1u,
                           a.wait_ns < dev::kDrainNs ? a.wait_ns : dev::kDrainNs);
        if (a.late_wait) asm volatile("griddepcontrol.wait;" ::: "memory");
    };

    while (true) {
        if (!dev::mbar_wait(full0 + 8 * cstage, cphase, a.wait_ns)) {
            timed_out();
            return;
        }
        if (trace && seq == 0 && lane == 0) trace[2] = dev::global_timer();
        const StageHdr hd = hdr[cstage];
        if (hd.flags & kHdrStop) {
            if (trace && lane == 0) trace[3] = dev::global_timer();
            break;
        }
        const int sA = cstage;
        advance();
        int sB = sA;
        int validB = 0;
        int32_t last_flags = hd.flags;
        const bool pair = (hd.flags & kHdrPair) != 0;
        if (pair) {
            if (!dev::mbar_wait(full0 + 8 * cstage, cphase, a.wait_ns)) {
                timed_out();
                return;
            }
            const StageHdr hb = hdr[cstage];
            sB = cstage;
            validB = hb.valid;
            last_flags = hb.flags;
            advance();
        }
        const unsigned char *stA = ring + static_cast<size_t>(sA) * a.stage_bytes;
        const unsigned char *stB = ring + static_cast<size_t>(sB) * a.stage_bytes;
        const bool slow = TIERED && (hd.flags & kHdrSlow);

        if (hd.flags & kHdrFirst) {
            // New item: query fragments (B operand, N = head g of this KV head) and state.
            item_slow = slow;
            const unsigned char *qs = stA + 2 * L::KB;
#pragma unroll
            for (int j = 0; j < KSTEPS; ++j) {
                if (g < a.G) {
                    if (!slow) {
                        qf[j][0] = *reinterpret_cast<const uint32_t *>(qs + (g * D + 16 * j + 2 * t) * 2);
                        qf[j][1] = *reinterpret_cast<const uint32_t *>(qs + (g * D + 16 * j + 2 * t + 8) * 2);
                    }
                } else {
                    qf[j][0] = 0u;
                    qf[j][1] = 0u;
                }
            }
            if (slow) {
                // INT8 tier: q of head g as s_q * (q1 + q2 / 254) with int8 digits q1, q2
                // (|error| <= max|q| / 64516 per element); B fragments of mma.m16n8k32.s8:
                // qf[jj] = q1 and qf[KS/2 + jj] = q2 at d = 32 jj + 4t + (0..3 | 16..19).
                float qv[KSTEPS / 2][8];
                float amax = 0.f;
#pragma unroll
                for (int jj = 0; jj < KSTEPS / 2; ++jj) {
                    if (g < a.G) {
                        const uint2 v0 = *reinterpret_cast<const uint2 *>(qs + (g * D + 32 * jj + 4 * t) * 2);
                        const uint2 v1 = *reinterpret_cast<const uint2 *>(qs + (g * D + 32 * jj + 16 + 4 * t) * 2);
                        qv[jj][0] = dev::bf16_lo(v0.x); qv[jj][1] = dev::bf16_hi(v0.x);
                        qv[jj][2] = dev::bf16_lo(v0.y); qv[jj][3] = dev::bf16_hi(v0.y);
                        qv[jj][4] = dev::bf16_lo(v1.x); qv[jj][5] = dev::bf16_hi(v1.x);
                        qv[jj][6] = dev::bf16_lo(v1.y); qv[jj][7] = dev::bf16_hi(v1.y);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) qv[jj][e] = 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(qv[jj][e]));
                }
                amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 1));
                amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 2));
                const float inv = amax > 0.f ? 127.f / amax : 0.f;
                const float sq = amax / 127.f;
                int32_t sum1 = 0, sum2 = 0;  // this lane's digit sums (INT4 offset correction)
#pragma unroll
                for (int jj = 0; jj < KSTEPS / 2; ++jj) {
                    uint32_t d1[2] = {0u, 0u}, d2[2] = {0u, 0u};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float y = qv[jj][e] * inv;
                        const int c1 = max(-127, min(127, __float2int_rn(y)));
                        const int c2 = max(-127, min(127, __float2int_rn((y - static_cast<float>(c1)) * 254.f)));
                        sum1 += c1;
                        sum2 += c2;
                        d1[e >> 2] |= (static_cast<uint32_t>(c1) & 0xFFu) << (8 * (e & 3));
                        d2[e >> 2] |= (static_cast<uint32_t>(c2) & 0xFFu) << (8 * (e & 3));
                    }
                    qf[jj][0] = d1[0];
                    qf[jj][1] = d1[1];
                    qf[KSTEPS / 2 + jj][0] = d2[0];
                    qf[KSTEPS / 2 + jj][1] = d2[1];
                }
                // per-head factor of the integer scores: s_q * scale * log2(e) / 254
                const float sqf = sq * (a.scale_log2 * (1.f / 254.f));
                ps.sq0 = __shfl_sync(FULL, sqf, 8 * t);      // head 2t lives in lanes 4 * 2t + ...
                ps.sq1 = __shfl_sync(FULL, sqf, 8 * t + 4);  // head 2t+1
                if (SB == 4) {
                    // the four lanes of head g hold all D of its digits
                    sum1 += __shfl_xor_sync(FULL, sum1, 1);
                    sum1 += __shfl_xor_sync(FULL, sum1, 2);
                    sum2 += __shfl_xor_sync(FULL, sum2, 1);
                    sum2 += __shfl_xor_sync(FULL, sum2, 2);
                    const int32_t corr = 8 * (254 * sum1 + sum2);
                    ps.k0 = __shfl_sync(FULL, corr, 8 * t);
                    ps.k1 = __shfl_sync(FULL, corr, 8 * t + 4);
                }
            }
#pragma unroll
            for (int i = 0; i < KSTEPS; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
            ps.reset();
        }

        const uint32_t aA = dev::smem_addr(stA), aB = dev::smem_addr(stB);
        if (!slow) {
            if (pair) {
                const uint32_t sa[2] = {aA, aB};
                const int va[2] = {hd.valid, validB};
                consume_pages<D, 2, false>(sa, va, qf, o, ps, offK, offV, off8, a.scale_log2, lane,
                                           a.token_scores, hd.tpos, a.G);
            } else {
                const uint32_t sa[1] = {aA};
                const int va[1] = {hd.valid};
                consume_pages<D, 1, false>(sa, va, qf, o, ps, offK, offV, off8, a.scale_log2, lane,
                                           a.token_scores, hd.tpos, a.G);
            }
        } else if (TIERED) {
            if (pair) {
                const uint32_t sa[2] = {aA, aB};
                const int va[2] = {hd.valid, validB};
                consume_pages<D, 2, true, SB>(sa, va, qf, o, ps, offK, offV, off8, a.scale_log2, lane);
            } else {
                const uint32_t sa[1] = {aA};
                const int va[1] = {hd.valid};
                consume_pages<D, 1, true, SB>(sa, va, qf, o, ps, offK, offV, off8, a.scale_log2, lane);
            }
        }
        __syncwarp();
        if (lane == 0) {
            dev::mbar_arrive(empty0 + 8 * sA);
            if (pair) dev::mbar_arrive(empty0 + 8 * sB);
        }

        if (last_flags & kHdrLast) {
            // ---- finish the item ----
            float E0 = ps.le0, E1 = ps.le1, R0 = ps.lr0, R1 = ps.lr1;
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                E0 += __shfl_xor_sync(FULL, E0, off);
                E1 += __shfl_xor_sync(FULL, E1, off);
                R0 += __shfl_xor_sync(FULL, R0, off);
                R1 += __shfl_xor_sync(FULL, R1, off);
            }
            if (TIERED && item_slow) {
                // the V codes entered P V with their offsets (see i8pair_to_f16, nib_lo_f16):
                // remove offset * sum(p') per head, and the x16 of the INT4 high-nibble tiles
                float W0 = ps.w0, W1 = ps.w1;
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    W0 += __shfl_xor_sync(FULL, W0, off);
                    W1 += __shfl_xor_sync(FULL, W1, off);
                }
#pragma unroll
                for (int i = 0; i < KSTEPS; ++i) {
                    const bool hi4 = SB == 4 && i >= KSTEPS / 2;
                    const float f = hi4 ? 1.f / 16.f : 1.f;
                    const float off = SB == 4 ? (hi4 ? dev::kV4HiOffset : dev::kV4LoOffset) : dev::kV8Offset;
                    o[i][0] = o[i][0] * f - off * W0;
                    o[i][2] = o[i][2] * f - off * W0;
                    o[i][1] = o[i][1] * f - off * W1;
                    o[i][3] = o[i][3] * f - off * W1;
                }
            }
            const float inv0 = R0 > 0.f ? 1.f / R0 : 0.f, inv1 = R1 > 0.f ? 1.f / R1 : 0.f;
            constexpr float kLn2 = 0.69314718055994530942f;
            const float lse0 = E0 > 0.f ? (ps.m0 + dev::lg2(E0)) * kLn2 : -INFINITY;
            const float lse1 = E1 > 0.f ? (ps.m1 + dev::lg2(E1)) * kLn2 : -INFINITY;
            const int32_t b = hd.bh / a.Hkv, h = hd.bh - b * a.Hkv;
            const int n0 = 2 * t, n1 = 2 * t + 1;
            if (hd.slot < 0) {
                const int64_t obase = (static_cast<int64_t>(b) * a.Hq + static_cast<int64_t>(h) * a.G) * D;
                __nv_bfloat16 *ob = a.out_f32 ? nullptr : a.out + obase;
                float *of = a.out_f32 ? a.out_f32 + obase : nullptr;
#pragma unroll
                for (int i = 0; i < KSTEPS; ++i) {
                    int dlo, dhi;
                    if (!item_slow) {
                        dlo = 16 * i + g;
                        dhi = dlo + 8;
                    } else {
                        dlo = 16 * i + 2 * g;
                        dhi = dlo + 1;
                    }
                    if (of) {
                        if (n0 < a.G) {
                            of[n0 * D + dlo] = o[i][0] * inv0;
                            of[n0 * D + dhi] = o[i][2] * inv0;
                        }
                        if (n1 < a.G) {
                            of[n1 * D + dlo] = o[i][1] * inv1;
                            of[n1 * D + dhi] = o[i][3] * inv1;
                        }
                    } else {
                        if (n0 < a.G) {
                            ob[n0 * D + dlo] = __float2bfloat16_rn(o[i][0] * inv0);
                            ob[n0 * D + dhi] = __float2bfloat16_rn(o[i][2] * inv0);
                        }
                        if (n1 < a.G) {
                            ob[n1 * D + dlo] = __float2bfloat16_rn(o[i][1] * inv1);
                            ob[n1 * D + dhi] = __float2bfloat16_rn(o[i][3] * inv1);
                        }
                    }
                }
                if (g == 0) {
                    float *lb = a.lse + static_cast<int64_t>(b) * a.Hq + static_cast<int64_t>(h) * a.G;
                    if (n0 < a.G) lb[n0] = lse0;
                    if (n1 < a.G) lb[n1] = lse1;
                }
            } else {
                float *po = a.part_o + static_cast<int64_t>(hd.slot) * a.G * D;
#pragma unroll
                for (int i = 0; i < KSTEPS; ++i) {
                    int dlo, dhi;
                    if (!item_slow) {
                        dlo = 16 * i + g;
                        dhi = dlo + 8;
                    } else {
                        dlo = 16 * i + 2 * g;
                        dhi = dlo + 1;
                    }
                    if (n0 < a.G) {
                        po[n0 * D + dlo] = o[i][0] * inv0;
                        po[n0 * D + dhi] = o[i][2] * inv0;
                    }
                    if (n1 < a.G) {
                        po[n1 * D + dlo] = o[i][1] * inv1;
                        po[n1 * D + dhi] = o[i][3] * inv1;
                    }
                }
                if (g == 0) {
                    float *pl = a.part_lse + static_cast<int64_t>(hd.slot) * a.G;
                    if (n0 < a.G) pl[n0] = lse0;
                    if (n1 < a.G) pl[n1] = lse1;
                }
            }
        }
    }
    if (trace && lane == 0) trace[4] = dev::global_timer();
    if (a.late_wait) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ------------------------------------------------------------------------------------------
// Prefix cascade kernel (5th-generation tensor cores): one CTA per cascade unit, a run of pages
// shared by up to two tiles of 128 query rows (each row one (reader, query head) pair).
//   warps 0-3 / 4-7: softmax of tile 0 / 1; thread i of a warpgroup owns query row i, which is
//                    lane i of tensor memory, so a row's max and sums need no shuffles
//   warps 8 / 9:     MMA issue of tile 0 / 1 (lane 0); warp 8 also allocates tensor memory
//   warp 10:         producer: page ids 32 at a time, 2-D TMA loads of K and V, 4 pages (64
//                    tokens) per block, into a ring of kTcStages blocks
// Per block and tile: S = Q K^T (M = 128 rows, N = 64 tokens, K = D; both operands K-major,
// 128-byte swizzled, S in tensor memory); the softmax reads S with tcgen05.ld, keeps the
// running max (lazy rescale: the max moves only when a block exceeds it by 2^8; then O is
// read, scaled and written back in tensor memory) and writes P as bf16 pairs back over the
// first 32 columns of the same S buffer with tcgen05.st; O += P V (M = 128, N = D, K = 16
// tokens per page; A = P from tensor memory, V the MN-major shared-memory operand, as stored).
// The two tiles alternate, so one tile's softmax overlaps the other's MMAs. Each reader's
// rows end as a normalised partial (o, lse) in its slot, merged with the head's other
// partials by the merge kernel.
// Tensor memory (512 columns): tile t holds two S / P buffers in columns [256t, 256t + 128)
// and O in [256t + 128, 256t + 128 + D). Shared memory: the two Q tiles, then the K/V ring.
// ------------------------------------------------------------------------------------------
struct CascadeArgs {
    const CascadeUnit *units;
    int32_t G, Hq, Hkv;
    float scale_log2;
    const __nv_bfloat16 *q;
    const int32_t *table;
    const int64_t *head_off;
    const int32_t *kv_len_dev;
    int64_t num_pages;
    float *part_o;
    float *part_lse;
    uint32_t *err;
    uint64_t wait_ns;
};

namespace tc {

// 32 lanes x 64 consecutive columns of fp32 from tensor memory (lane = the warp's quarter).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
                 :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Shared-memory matrix descriptor of a 128-byte-swizzled operand (atoms of 8 rows x 128 bytes,
// 1024-byte aligned): start address, leading byte offset, stride byte offset (8-row groups),
// the descriptor version of this architecture (1) and the swizzle mode (2 = 128 bytes).
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) |
           (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, A K-major, B K-major
// (b_mn = 0) or MN-major (b_mn = 1), N and M.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t n, uint32_t m, uint32_t b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn << 16) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

__device__ __forceinline__ void mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                    uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

// As mma, with the A operand in tensor memory at a_tmem (M rows on the lanes, K along the
// columns, two 16-bit elements per 32-bit column).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        :: "r"(d_tmem), "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives on the mbarrier once every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(bar) : "memory");
}

}  // namespace tc

constexpr int kTcRows = 128;               // rows per tile = tensor-memory lanes
constexpr int kTcThreads = 11 * 32;        // 8 softmax warps, 2 MMA warps, 1 producer warp
constexpr int kTcStages = 5;               // K/V blocks in flight
constexpr uint32_t kTcCols = 512;          // tensor-memory columns of the CTA

template <int D>
struct TcLayout {
    static constexpr int kHalves = D / 64;                  // 64-element (128-byte) column halves
    static constexpr int kQTile = kTcRows * D * 2;          // one tile of Q
    static constexpr int kKBlock = 64 * D * 2;              // 64 tokens of K
    static constexpr int kStage = 2 * kKBlock;              // K then V
    static constexpr int kQ = 0;
    static constexpr int kKV = kQ + 2 * kQTile;
    static constexpr int kBars = kKV + kTcStages * kStage;  // mbarriers, then the TMEM address
    static constexpr int kBytes = kBars + 256;
};

template <int D>
constexpr int cascade_smem_bytes() {
    return 1024 + TcLayout<D>::kBytes;
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    cascade_kernel(const __grid_constant__ CascadeArgs a, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v) {
    using TL = TcLayout<D>;
    constexpr int KS = D / 16;  // k-steps of S = Q K^T
    constexpr unsigned FULL = 0xffffffffu;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = dev::smem_addr(smem);
    // mbarriers: kv_full[S], kv_empty[S], q_full, then per tile t and buffer b (index 2t + b):
    // s_full[4], p_full[4], o_done[4]; then drain[2]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + TL::kBars);
    const uint32_t bar0 = dev::smem_addr(bars);
    const uint32_t kv_full = bar0, kv_empty = bar0 + 8 * kTcStages, q_full = bar0 + 16 * kTcStages;
    const uint32_t s_full = q_full + 8, p_full = s_full + 32, o_done = p_full + 32, drain = o_done + 32;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + TL::kBars + 8 * (2 * kTcStages + 15));
    volatile int32_t *abort_flag = reinterpret_cast<volatile int32_t *>(tmem_slot + 1);

    const CascadeUnit *u = a.units + blockIdx.x;
    const int32_t h = u->h, pb = u->pos_begin, pe = u->pos_end, nr = u->n_readers;
    const int32_t G = a.G;
    const int32_t npages = pe - pb;
    const int32_t nblocks = (npages + 3) / 4;
    const int32_t ntiles = nr * G > kTcRows ? 2 : 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int st = 0; st < kTcStages; ++st) {
            dev::mbar_init(kv_full + 8 * st, 1);
            dev::mbar_init(kv_empty + 8 * st, ntiles);
        }
        dev::mbar_init(q_full, 4 * ntiles);
        for (int k = 0; k < 4; ++k) {
            dev::mbar_init(s_full + 8 * k, 1);
            dev::mbar_init(p_full + 8 * k, 4);
            dev::mbar_init(o_done + 8 * k, 1);
        }
        dev::mbar_init(drain, 1);
        dev::mbar_init(drain + 8, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 8) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(dev::smem_addr(tmem_slot)), "r"(kTcCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;
    // The previous kernel in the stream completes first; then the next one may launch.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    auto timed_out = [&]() {
        atomicOr(a.err, kErrTimeout);
        *abort_flag = 1;
    };

    if (warp == 10) {
        // ================================ producer warp ================================
        const int32_t *row = a.table + a.head_off[static_cast<int64_t>(u->reader[0]) * a.Hkv + h] + pb;
        int32_t ids = lane < npages ? __ldg(row + lane) : -1;
        int32_t ids_next = 32 + lane < npages ? __ldg(row + 32 + lane) : -1;
        int32_t issued = 0;
        for (int32_t blk = 0; blk < nblocks; ++blk) {
            if (blk == 1) {
                // every reader's length still covers the run (checked once the copies are going)
                bool bad = false;
                for (int32_t r = lane; r < nr; r += 32)
                    bad |= a.kv_len_dev[static_cast<int64_t>(u->reader[r]) * a.Hkv + h] < pe * 16;
                if (__any_sync(FULL, bad) && lane == 0) atomicOr(a.err, kErrPlan);
            }
            const int st = blk % kTcStages;
            const uint32_t ph = static_cast<uint32_t>(blk / kTcStages) & 1u;
            int32_t stop = 0;
            if (lane == 0 && (!dev::mbar_wait(kv_empty + 8 * st, ph ^ 1u, a.wait_ns) || *abort_flag)) {
                timed_out();
                stop = 1;
            }
            if (__shfl_sync(FULL, stop, 0)) break;
            const int32_t np = min(4, npages - 4 * blk);
            const uint32_t kv = sbase + TL::kKV + st * TL::kStage;
            if (lane == 0) dev::mbar_arrive_expect_tx(kv_full + 8 * st, static_cast<uint32_t>(np) * 2u * 16u * D * 2u);
            // lane k < np loads page 4 blk + k (its ids block starts at a multiple of 32 pages,
            // and 4 blk .. 4 blk + 3 never straddle one)
            if (blk > 0 && ((4 * blk) & 31) == 0) {
                ids = ids_next;
                ids_next = 4 * blk + 32 + lane < npages ? __ldg(row + 4 * blk + 32 + lane) : -1;
            }
            int64_t pid = __shfl_sync(FULL, ids, (4 * blk + (lane & 3)) & 31);
            __syncwarp();
            if (lane < np) {
                if (pid < 0 || pid >= a.num_pages) {
                    atomicOr(a.err, kErrBadPage);
                    pid = 0;  // a page of the pool; the result is flagged as wrong
                }
                const int32_t y = static_cast<int32_t>(pid * 16);
#pragma unroll
                for (int hf = 0; hf < TL::kHalves; ++hf) {
                    dev::tma_load_2d(kv + hf * (TL::kKBlock / TL::kHalves) + lane * 2048, &tm_k, hf * 64, y, kv_full + 8 * st);
                    dev::tma_load_2d(kv + TL::kKBlock + hf * (TL::kKBlock / TL::kHalves) + lane * 2048, &tm_v, hf * 64, y,
                                     kv_full + 8 * st);
                }
            }
            __syncwarp();
            issued = blk + 1;
        }
        if (nblocks <= 1) {
            bool bad = false;
            for (int32_t r = lane; r < nr; r += 32)
                bad |= a.kv_len_dev[static_cast<int64_t>(u->reader[r]) * a.Hkv + h] < pe * 16;
            if (__any_sync(FULL, bad) && lane == 0) atomicOr(a.err, kErrPlan);
        }
        // No copy may be in flight when the CTA exits: wait for the last block of every stage.
        if (lane == 0)
            for (int32_t b = issued - kTcStages < 0 ? 0 : issued - kTcStages; b < issued; ++b)
                dev::mbar_wait(kv_full + 8 * (b % kTcStages), static_cast<uint32_t>(b / kTcStages) & 1u,
                               a.wait_ns < dev::kDrainNs ? a.wait_ns : dev::kDrainNs);
        return;
    }

    if (warp == 8 || warp == 9) {
        // ========================= MMA warps (tile 0: warp 8, tile 1: warp 9) =========================
        // S(blk) goes to tensor-memory buffer blk & 1 and is issued before PV(blk - 1), so the
        // next block's scores are ready when the softmax finishes a block. The softmax writes
        // P(blk) as bf16 pairs over the first 32 columns of S(blk)'s buffer, and PV(blk) takes it
        // from there as its A operand; S(blk + 2), which reuses the buffer, is issued by this
        // thread after PV(blk), and the MMAs of one thread run in issue order.
        const int t = warp - 8;
        if (lane == 0 && t < ntiles) {
            const uint32_t id_s = tc::idesc_bf16(64, kTcRows, 0);
            const uint32_t id_o = tc::idesc_bf16(D, kTcRows, 1);
            const uint32_t q = sbase + TL::kQ + t * TL::kQTile;
            bool ok = dev::mbar_wait(q_full, 0, a.wait_ns);
            tc::fence_after();
            auto issue_o = [&](int32_t blk) {
                const uint32_t kv = sbase + TL::kKV + (blk % kTcStages) * TL::kStage + TL::kKBlock;
                const uint32_t pt = tmem + 256 * t + 64 * (blk & 1);  // P(blk): 8 columns per 16 tokens
                const int32_t np = min(4, npages - 4 * blk);
                for (int32_t k = 0; k < np; ++k)
                    tc::mma_ts(tmem + 256 * t + 128, pt + 8 * k,
                               tc::sdesc(kv + k * 2048, TL::kKBlock / TL::kHalves, 1024), id_o, blk > 0 || k > 0);
                tc::commit(o_done + 8 * (2 * t + (blk & 1)));
                tc::commit(kv_empty + 8 * (blk % kTcStages));
            };
            for (int32_t blk = 0; ok && blk <= nblocks; ++blk) {
                if (blk < nblocks) {
                    const int st = blk % kTcStages;
                    ok = dev::mbar_wait(kv_full + 8 * st, static_cast<uint32_t>(blk / kTcStages) & 1u, a.wait_ns) &&
                         !*abort_flag;
                    tc::fence_after();
                    if (!ok) break;
                    const uint32_t kv = sbase + TL::kKV + st * TL::kStage;
#pragma unroll
                    for (int k = 0; k < KS; ++k) {
                        const uint32_t hf = k / 4, off = (k % 4) * 32;
                        tc::mma(tmem + 256 * t + 64 * (blk & 1),
                                tc::sdesc(q + hf * (kTcRows * 128) + off, 16, 1024),
                                tc::sdesc(kv + hf * (TL::kKBlock / TL::kHalves) + off, 16, 1024), id_s, k > 0);
                    }
                    tc::commit(s_full + 8 * (2 * t + (blk & 1)));
                }
                if (blk >= 1) {
                    const int32_t pbk = blk - 1;
                    ok = dev::mbar_wait(p_full + 8 * (2 * t + (pbk & 1)), static_cast<uint32_t>(pbk >> 1) & 1u, a.wait_ns) &&
                         !*abort_flag;
                    tc::fence_after();
                    if (!ok) break;
                    issue_o(pbk);
                }
            }
            if (!ok) timed_out();
            // every MMA this thread issued has finished before tensor memory is released
            tc::commit(drain + 8 * t);
            dev::mbar_wait(drain + 8 * t, 0, a.wait_ns < dev::kDrainNs ? a.wait_ns : dev::kDrainNs);
        }
        __syncwarp();
    } else {
        // ================================ softmax warpgroups ================================
        const int t = warp >> 2, qd = warp & 3;
        const int i = 32 * qd + lane;                 // row of the tile = tensor-memory lane
        const int r = kTcRows * t + i;                // row of the unit
        const bool active = t < ntiles;
        const bool valid = r < nr * G;
        const uint32_t lanes = static_cast<uint32_t>(32 * qd) << 16;
        const uint32_t t_s = tmem + lanes + 256 * t, t_o = t_s + 128;
        float m = -INFINITY, le = 0.f;
        if (active) {
            // Q row -> the tile's swizzled K-major layout (zeros for rows past the readers)
            const uint32_t qrow = sbase + TL::kQ + t * TL::kQTile + i * 128;
            const uint4 *src = valid ? reinterpret_cast<const uint4 *>(
                                           a.q + (static_cast<int64_t>(u->reader[r / G]) * a.Hq + h * G + r % G) * D)
                                     : nullptr;
            // every load of the row in flight before the first store (an asm store with a
            // memory clobber would otherwise hold each next load back: D/8 serial round trips)
            uint4 qv[D / 8];
#pragma unroll
            for (int c = 0; c < D / 8; ++c) qv[c] = src ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const uint32_t addr = qrow + (c / 8) * (kTcRows * 128) + (((c % 8) ^ (i & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                             :: "r"(addr), "r"(qv[c].x), "r"(qv[c].y), "r"(qv[c].z), "r"(qv[c].w) : "memory");
            }
            tc::fence_async_smem();
            __syncwarp();
            if (lane == 0) dev::mbar_arrive(q_full);

            bool ok = true;
            for (int32_t blk = 0; blk < nblocks; ++blk) {
                const int bf = blk & 1;
                const uint32_t ph = static_cast<uint32_t>(blk >> 1) & 1u;   // phase of buffer bf's barriers
                ok = dev::mbar_wait(s_full + 8 * (2 * t + bf), ph, a.wait_ns) && !*abort_flag;
                if (!__all_sync(FULL, ok)) { ok = false; break; }
                tc::fence_after();
                uint32_t sr[64];
                tc::tmem_ld64(t_s + 64 * bf, sr);
                tc::tmem_wait_ld();
                const int32_t nv = 16 * min(4, npages - 4 * blk);    // valid tokens of the block
                // row max of the raw scores (the scale is positive), 8 independent chains
                float mr[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) mr[c] = -INFINITY;
                if (nv == 64) {
#pragma unroll
                    for (int c = 0; c < 64; ++c) mr[c & 7] = fmaxf(mr[c & 7], __uint_as_float(sr[c]));
                } else {
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (c < nv) mr[c & 7] = fmaxf(mr[c & 7], __uint_as_float(sr[c]));
                }
                const float mx = fmaxf(fmaxf(fmaxf(mr[0], mr[1]), fmaxf(mr[2], mr[3])),
                                       fmaxf(fmaxf(mr[4], mr[5]), fmaxf(mr[6], mr[7]))) * a.scale_log2;
                const bool up = mx > m + 8.f;
                if (__any_sync(FULL, up)) {
                    const float mn = up ? mx : m;
                    const float c0 = !up ? 1.f : (m == -INFINITY ? 0.f : dev::ex2(m - mn));
                    if (blk > 0) {
                        // O holds PV(0 .. blk - 1): wait for PV(blk - 1), then scale it in place
                        ok = dev::mbar_wait(o_done + 8 * (2 * t + (bf ^ 1)), static_cast<uint32_t>((blk - 1) >> 1) & 1u,
                                            a.wait_ns) && !*abort_flag;
                        if (!__all_sync(FULL, ok)) { ok = false; break; }
                        tc::fence_after();
#pragma unroll 1
                        for (int ch = 0; ch < D / 32; ++ch) {
                            uint32_t o[32];
                            tc::tmem_ld32(t_o + 32 * ch, o);
                            tc::tmem_wait_ld();
#pragma unroll
                            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * c0);
                            tc::tmem_st32(t_o + 32 * ch, o);
                        }
                        tc::tmem_wait_st();
                    }
                    le *= c0;
                    m = mn;
                }
                // p = 2^(s * scale - m): one FFMA and one ex2 per score; 8 partial sums. P goes
                // to the first 32 columns of this S buffer (bf16 pairs; the scores are in
                // registers), the A operand of PV(blk).
                float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                const float nm = -m;
                uint32_t pw[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int c = 2 * e;
                    float p0 = dev::ex2(fmaf(__uint_as_float(sr[c]), a.scale_log2, nm));
                    float p1 = dev::ex2(fmaf(__uint_as_float(sr[c + 1]), a.scale_log2, nm));
                    if (nv < 64) {
                        p0 = c < nv ? p0 : 0.f;
                        p1 = c + 1 < nv ? p1 : 0.f;
                    }
                    ls[e & 3] += p0;
                    ls[4 + (e & 3)] += p1;
                    pw[e] = dev::pack_bf16(p0, p1);
                }
                le += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
                tc::tmem_st32(t_s + 64 * bf, pw);
                tc::tmem_wait_st();
                tc::fence_before();
                __syncwarp();
                if (lane == 0) dev::mbar_arrive(p_full + 8 * (2 * t + bf));
            }
            // all of PV(0 .. nblocks - 1) are done: wait for the last two
            for (int32_t b = nblocks - 2 < 0 ? 0 : nblocks - 2; ok && b < nblocks; ++b) {
                ok = dev::mbar_wait(o_done + 8 * (2 * t + (b & 1)), static_cast<uint32_t>(b >> 1) & 1u, a.wait_ns);
                ok = __all_sync(FULL, ok);
            }
            tc::fence_after();
            if (!ok) {
                if (lane == 0) timed_out();
            } else {
                // out row = O / le (partial), lse = (m + log2 le) ln 2. The warp's 32 rows leave
                // through shared memory (the tile's Q region: its last S MMA ran before its last
                // PV, which is done), so that each store writes whole 128-byte row segments (8
                // lanes a row, 4 rows a store) instead of a 16-byte piece of each of 32 rows: 8x
                // fewer L2 transactions.
                const float inv = le > 0.f ? 1.f / le : 0.f;
                const uint32_t stg = sbase + TL::kQ + static_cast<uint32_t>(t * TL::kQTile + qd * 4096);  // 32 rows x 128 B
                float *dst[8];  // rows 4k + lane / 8 of this warp (null past the readers)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int rr = kTcRows * t + 32 * qd + 4 * k + (lane >> 3);
                    dst[k] = rr < nr * G ? a.part_o + (static_cast<int64_t>(u->slot[rr / G]) * G + rr % G) * D + 4 * (lane & 7)
                                         : nullptr;
                }
#pragma unroll 1
                for (int ch = 0; ch < D / 32; ++ch) {
                    uint32_t o[32];
                    tc::tmem_ld32(t_o + 32 * ch, o);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8) {
                        const uint32_t addr = stg + lane * 128 + ((c8 ^ (lane & 7)) << 4);
                        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};"
                                     :: "r"(addr), "f"(__uint_as_float(o[4 * c8]) * inv),
                                        "f"(__uint_as_float(o[4 * c8 + 1]) * inv), "f"(__uint_as_float(o[4 * c8 + 2]) * inv),
                                        "f"(__uint_as_float(o[4 * c8 + 3]) * inv)
                                     : "memory");
                    }
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int j = 4 * k + (lane >> 3), c8 = lane & 7;
                        float4 v;
                        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                     : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                                     : "r"(stg + j * 128 + ((c8 ^ (j & 7)) << 4))
                                     : "memory");
                        if (dst[k]) *reinterpret_cast<float4 *>(dst[k] + 32 * ch) = v;
                    }
                    __syncwarp();
                }
                if (valid) {
                    constexpr float kLn2 = 0.69314718055994530942f;
                    a.part_lse[static_cast<int64_t>(u->slot[r / G]) * G + r % G] =
                        le > 0.f ? (m + dev::lg2(le)) * kLn2 : -INFINITY;
                }
            }
        }
    }
    // Warps 0-9 meet before tensor memory is released (the producer may have left already).
    tc::fence_before();
    asm volatile("bar.sync 1, %0;" :: "r"(10 * 32) : "memory");
    tc::fence_after();
    if (warp == 8) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTcCols) : "memory");
}

// ------------------------------------------------------------------------------------------
// Lean decode kernel: whole-head plans of short heads (a tiny batch, where a step is the latency
// of one launch and a few dependent memory reads, not bandwidth). CTA i < B*Hkv handles
// (sequence, KV head) i with all its G query heads; no copy pipeline, tensor map or
// shared-memory ring to set up, so the critical path is: lengths and row offset, page ids,
// K/V rows (all of a chunk's loads in flight at once), arithmetic, one merge through shared
// memory, the output.
//   Lanes: a token row of D bf16 is D/8 16-byte slices; LPT = D/8 lanes hold one token (lane
//   sub = lane % LPT has dims [8 sub, 8 sub + 8)), so a warp covers TPW = 32/LPT tokens per
//   round; R rounds per chunk (fewer for larger G: the per-lane state grows with G).
//   Scores: fp32 dot products of the 8-dim slices summed over the LPT lanes by xor-shuffles,
//   in log2 units; each lane keeps its own running max, sum and output slice over its tokens
//   (the online-normaliser identity), rescaled once per chunk.
//   Merge: the TPW token groups of a warp by xor-shuffles, then the warps through shared memory
//   (fixed order, so results are deterministic); out = O / L, lse = ln 2 (M + log2 L).
// ------------------------------------------------------------------------------------------
struct LeanArgs {
    int32_t Hq, Hkv;
    float scale_log2;
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k_pages, *v_pages;
    const int32_t *table;
    const int64_t *head_off;
    const int32_t *group_of_head;
    const int64_t *group_off;
    int32_t n_groups;
    const int32_t *kv_len_dev;
    const int32_t *planned;          // [B*Hkv] the plan's lengths
    int64_t num_pages;
    __nv_bfloat16 *out;
    float *out_f32;
    float *lse;
    uint32_t *err;
    int32_t early_prologue;
};

template <int D, int G>
__global__ void __launch_bounds__(kLeanWarps * 32) lean_decode_kernel(const __grid_constant__ LeanArgs a) {
    constexpr int LPT = D / 8;
    constexpr int TPW = 32 / LPT;
    constexpr int R = G <= 2 ? 8 : (G == 4 ? 4 : 2);
    constexpr int CHUNK = kLeanWarps * TPW * R;
    constexpr unsigned FULL = 0xffffffffu;
    __shared__ float red_o[kLeanWarps][G][D];
    __shared__ float red_m[kLeanWarps][G];
    __shared__ float red_l[kLeanWarps][G];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane % LPT, tig = lane / LPT;
    const int32_t bh = blockIdx.x;
    const int32_t b = bh / a.Hkv, h = bh - b * a.Hkv;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!a.early_prologue) asm volatile("griddepcontrol.wait;" ::: "memory");

    // Metadata: planned and current length, row offset and the whole table's bounds (all
    // independent loads); the row is first checked against the whole table, which is enough to
    // read its page ids safely, and against its own group's table while those loads are in flight.
    const int32_t n = a.planned[bh];
    const int32_t n_dev = a.kv_len_dev[bh];
    const int64_t row = a.head_off[bh];
    const int32_t grp = a.group_of_head ? a.group_of_head[h] : 0;
    const int64_t t_lo = a.group_off[0], t_hi = a.group_off[a.n_groups];
    const int32_t npages = (n + 15) >> 4;
    const bool in_table = n == 0 || (row >= t_lo && row + npages <= t_hi);
    const int32_t n_eff = in_table ? n : 0;

    // Page ids of this lane's tokens of the first chunk (before the predecessor's wait: tables
    // only; queries and K/V after it).
    auto token_of = [&](int32_t c0, int r) { return c0 + (r * kLeanWarps + warp) * TPW + tig; };
    int32_t pid[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int32_t t = token_of(0, r);
        pid[r] = t < n_eff ? __ldg(a.table + row + (t >> 4)) : -1;
    }
    bool row_ok = in_table;
    if (a.group_of_head && n > 0) {
        if (grp >= 0 && grp < a.n_groups)
            row_ok = row_ok && row >= a.group_off[grp] && row + npages <= a.group_off[grp + 1];
        else
            row_ok = false;
    }
    if (threadIdx.x == 0) {
        if (n_dev != n) atomicOr(a.err, kErrPlan);
        if (!row_ok) atomicOr(a.err, kErrBadRow);
    }
    const int32_t n_use = row_ok ? n_eff : 0;  // a row outside its group's table reads nothing
    if (a.early_prologue) asm volatile("griddepcontrol.wait;" ::: "memory");

    float qf[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(
            a.q + (static_cast<int64_t>(b) * a.Hq + static_cast<int64_t>(h) * G + g) * D + 8 * sub));
        qf[g][0] = dev::bf16_lo(v.x); qf[g][1] = dev::bf16_hi(v.x);
        qf[g][2] = dev::bf16_lo(v.y); qf[g][3] = dev::bf16_hi(v.y);
        qf[g][4] = dev::bf16_lo(v.z); qf[g][5] = dev::bf16_hi(v.z);
        qf[g][6] = dev::bf16_lo(v.w); qf[g][7] = dev::bf16_hi(v.w);
    }
    float m[G], l[G], o[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) o[g][i] = 0.f;
    }

    for (int32_t c0 = 0; c0 < n_use; c0 += CHUNK) {
        if (c0 > 0) {
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int32_t t = token_of(c0, r);
                pid[r] = t < n_use ? __ldg(a.table + row + (t >> 4)) : -1;
            }
        }
        // every K and V slice of the chunk in flight before any arithmetic
        uint4 kr[R], vr[R];
        bool valid[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int32_t t = token_of(c0, r);
            valid[r] = false;
            kr[r] = make_uint4(0u, 0u, 0u, 0u);
            vr[r] = kr[r];
            if (t < n_use) {
                if (pid[r] < 0 || pid[r] >= a.num_pages) {
                    if (sub == 0) atomicOr(a.err, kErrBadPage);  // skipped, never read
                } else {
                    const int64_t off = (static_cast<int64_t>(pid[r]) * 16 + (t & 15)) * D + 8 * sub;
                    kr[r] = __ldg(reinterpret_cast<const uint4 *>(a.k_pages + off));
                    vr[r] = __ldg(reinterpret_cast<const uint4 *>(a.v_pages + off));
                    valid[r] = true;
                }
            }
        }
        float sc[R][G];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float kf[8];
            kf[0] = dev::bf16_lo(kr[r].x); kf[1] = dev::bf16_hi(kr[r].x);
            kf[2] = dev::bf16_lo(kr[r].y); kf[3] = dev::bf16_hi(kr[r].y);
            kf[4] = dev::bf16_lo(kr[r].z); kf[5] = dev::bf16_hi(kr[r].z);
            kf[6] = dev::bf16_lo(kr[r].w); kf[7] = dev::bf16_hi(kr[r].w);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) acc = fmaf(qf[g][i], kf[i], acc);
#pragma unroll
                for (int off = 1; off < LPT; off <<= 1) acc += __shfl_xor_sync(FULL, acc, off);
                sc[r][g] = valid[r] ? acc * a.scale_log2 : -INFINITY;
            }
        }
        // one rescale per chunk and head
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float mc = m[g];
#pragma unroll
            for (int r = 0; r < R; ++r) mc = fmaxf(mc, sc[r][g]);
            if (mc > m[g]) {
                const float al = m[g] == -INFINITY ? 0.f : dev::ex2(m[g] - mc);
                l[g] *= al;
#pragma unroll
                for (int i = 0; i < 8; ++i) o[g][i] *= al;
                m[g] = mc;
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float vf[8];
            vf[0] = dev::bf16_lo(vr[r].x); vf[1] = dev::bf16_hi(vr[r].x);
            vf[2] = dev::bf16_lo(vr[r].y); vf[3] = dev::bf16_hi(vr[r].y);
            vf[4] = dev::bf16_lo(vr[r].z); vf[5] = dev::bf16_hi(vr[r].z);
            vf[6] = dev::bf16_lo(vr[r].w); vf[7] = dev::bf16_hi(vr[r].w);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float pr = valid[r] ? dev::ex2(sc[r][g] - m[g]) : 0.f;
                l[g] += pr;
#pragma unroll
                for (int i = 0; i < 8; ++i) o[g][i] = fmaf(pr, vf[i], o[g][i]);
            }
        }
    }

    // Merge the warp's token groups (lanes that hold the same dims), then the warps.
#pragma unroll
    for (int off = LPT; off < 32; off <<= 1) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float mo = __shfl_xor_sync(FULL, m[g], off);
            const float lo2 = __shfl_xor_sync(FULL, l[g], off);
            const float M = fmaxf(m[g], mo);
            const float fa = m[g] == -INFINITY ? 0.f : dev::ex2(m[g] - M);
            const float fb = mo == -INFINITY ? 0.f : dev::ex2(mo - M);
            l[g] = l[g] * fa + lo2 * fb;
#pragma unroll
            for (int i = 0; i < 8; ++i) o[g][i] = o[g][i] * fa + __shfl_xor_sync(FULL, o[g][i], off) * fb;
            m[g] = M;
        }
    }
    if (tig == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int i = 0; i < 8; ++i) red_o[warp][g][8 * sub + i] = o[g][i];
            if (sub == 0) {
                red_m[warp][g] = m[g];
                red_l[warp][g] = l[g];
            }
        }
    }
    __syncthreads();
    constexpr float kLn2 = 0.69314718055994530942f;
    const int64_t obase = (static_cast<int64_t>(b) * a.Hq + static_cast<int64_t>(h) * G) * D;
    for (int idx = threadIdx.x; idx < G * D; idx += kLeanWarps * 32) {
        const int g = idx / D, d = idx - g * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kLeanWarps; ++w) M = fmaxf(M, red_m[w][g]);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kLeanWarps; ++w) {
                const float f = red_m[w][g] == -INFINITY ? 0.f : dev::ex2(red_m[w][g] - M);
                L = fmaf(red_l[w][g], f, L);
                O = fmaf(red_o[w][g][d], f, O);
            }
        }
        const float val = L > 0.f ? O / L : 0.f;
        if (a.out_f32)
            a.out_f32[obase + idx] = val;
        else
            a.out[obase + idx] = __float2bfloat16_rn(val);
        if (d == 0)
            a.lse[static_cast<int64_t>(b) * a.Hq + static_cast<int64_t>(h) * G + g] =
                L > 0.f ? (M + dev::lg2(L)) * kLn2 : -INFINITY;
    }
}

// ------------------------------------------------------------------------------------------
// Merge of split heads (log-sum-exp): one CTA per (split head, query row). Warp w owns the
// contiguous splits [w*k, (w+1)*k); it loads them 4 at a time (all loads in flight), keeps a
// running maximum and sum, and the warps' results are combined through shared memory in warp
// order, so the result does not depend on timing. Launched as a programmatic dependent of
// the decode kernel: it waits for that grid before reading.
// ------------------------------------------------------------------------------------------
template <int D, bool ROWS>
__global__ void __launch_bounds__(1024) split_merge_kernel(const MergeHead *mh, int64_t n_rows,
                                                           int32_t G, int32_t Hq, int32_t Hkv,
                                                           const float *part_o,
                                                           const float *part_lse,
                                                           __nv_bfloat16 *out, float *out_f32,
                                                           float *lse) {
    constexpr int VEC = D / 32;
    constexpr int U = 4;
    extern __shared__ float s_dyn[];  // [nw] maxima, [nw] sums, [nw][D] sums of V (nw > 1)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // Every CTA of this grid has started: the next kernel may be scheduled.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // ROWS: one warp per (split head, query row), several rows per CTA (heads of few splits);
    // else one CTA per row, its warps splitting the head's splits.
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = ROWS ? 1 : blockDim.x >> 5;
    const int64_t rid = ROWS ? static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp : blockIdx.x;
    if (rid >= n_rows) return;
    const MergeHead h = mh[rid / G];
    const int n = static_cast<int>(rid % G);
    const float *pl = part_lse + static_cast<int64_t>(h.first_slot) * G + n;
    const float *po = part_o + (static_cast<int64_t>(h.first_slot) * G + n) * D + lane * VEC;
    const int64_t pstride = static_cast<int64_t>(G) * D;
    const int k = (h.nsplit + nw - 1) / nw;
    const int j0 = (ROWS ? 0 : warp) * k, j1 = min(h.nsplit, j0 + k);

    float m = -INFINITY, sum = 0.f, acc[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) acc[c] = 0.f;
    for (int j = j0; j < j1; j += U) {
        float l[U], v[U][VEC];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const bool in = j + u < j1;
            l[u] = in ? pl[static_cast<int64_t>(j + u) * G] : -INFINITY;
            // the lane's VEC consecutive floats in one 8- or 16-byte load (rows of D floats)
            if constexpr (VEC == 4) {
                const float4 x = in ? *reinterpret_cast<const float4 *>(po + (j + u) * pstride)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                v[u][0] = x.x;
                v[u][1] = x.y;
                v[u][2] = x.z;
                v[u][3] = x.w;
            } else {
#pragma unroll
                for (int c = 0; c < VEC; ++c) v[u][c] = in ? po[(j + u) * pstride + c] : 0.f;
            }
        }
        float mc = m;
#pragma unroll
        for (int u = 0; u < U; ++u) mc = fmaxf(mc, l[u]);
        if (mc == -INFINITY) continue;
        const float r = m == -INFINITY ? 0.f : expf(m - mc);
        sum *= r;
#pragma unroll
        for (int c = 0; c < VEC; ++c) acc[c] *= r;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float w = expf(l[u] - mc);  // 0 for an empty or absent split
            sum += w;
#pragma unroll
            for (int c = 0; c < VEC; ++c) acc[c] += w * v[u][c];
        }
        m = mc;
    }
    const int32_t b = h.bh / Hkv, hh = h.bh - b * Hkv;
    const int64_t row = static_cast<int64_t>(b) * Hq + static_cast<int64_t>(hh) * G + n;
    if (!ROWS && nw > 1) {
        float *s_m = s_dyn, *s_s = s_dyn + nw;
        float(*s_acc)[D] = reinterpret_cast<float(*)[D]>(s_dyn + 2 * nw);
        if (lane == 0) {
            s_m[warp] = m;
            s_s[warp] = sum;
        }
#pragma unroll
        for (int c = 0; c < VEC; ++c) s_acc[warp][lane * VEC + c] = acc[c];
        __syncthreads();
        if (warp != 0) return;
        float M = -INFINITY;
        for (int w = 0; w < nw; ++w) M = fmaxf(M, s_m[w]);
        sum = 0.f;
#pragma unroll
        for (int c = 0; c < VEC; ++c) acc[c] = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < nw; ++w) {
                if (s_m[w] == -INFINITY) continue;
                const float r = expf(s_m[w] - M);
                sum += r * s_s[w];
#pragma unroll
                for (int c = 0; c < VEC; ++c) acc[c] += r * s_acc[w][lane * VEC + c];
            }
        }
        m = M;
    }
    const float inv = m == -INFINITY ? 0.f : 1.f / sum;
    if constexpr (VEC == 4) {
        if (out_f32) {
            *reinterpret_cast<float4 *>(out_f32 + row * D + lane * VEC) =
                make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        } else {
            // four bf16 in one 8-byte store
            *reinterpret_cast<uint2 *>(out + row * D + lane * VEC) =
                make_uint2(dev::pack_bf16(acc[0] * inv, acc[1] * inv), dev::pack_bf16(acc[2] * inv, acc[3] * inv));
        }
    } else {
#pragma unroll
        for (int c = 0; c < VEC; ++c) {
            if (out_f32)
                out_f32[row * D + lane * VEC + c] = acc[c] * inv;
            else
                out[row * D + lane * VEC + c] = __float2bfloat16_rn(acc[c] * inv);
        }
    }
    if (lane == 0) lse[row] = m == -INFINITY ? -INFINITY : m + logf(sum);
}

// Merge of split heads of 9..kLaneParts parts: one warp per (split head, query row), 8 rows
// per CTA. Lane j holds part j's lse; the row's maximum and the sum of the weights
// w_j = exp(l_j - max) are warp reductions; each lane then sums its D/32 columns over the parts,
// kPartBatch parts' loads at a time (all in flight), the weights broadcast from their lanes.
// Fewer dependent rounds than the multi-warp merge for heads of 9..32 parts, and no shared
// memory. The order of the sums is fixed, so the result does not depend on timing.
constexpr int kLaneParts = 32;
constexpr int kPartBatch = 16;

template <int D>
__global__ void __launch_bounds__(256) lane_merge_kernel(const MergeHead *mh, int64_t n_rows, int32_t G,
                                                         int32_t Hq, int32_t Hkv, const float *part_o,
                                                         const float *part_lse, __nv_bfloat16 *out,
                                                         float *out_f32, float *lse) {
    constexpr int VEC = D / 32;
    constexpr unsigned FULL = 0xffffffffu;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t rid = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (rid >= n_rows) return;
    const MergeHead h = mh[rid / G];
    const int n = static_cast<int>(rid % G);
    const int64_t pstride = static_cast<int64_t>(G) * D;
    const float *pl = part_lse + static_cast<int64_t>(h.first_slot) * G + n;
    const float *po = part_o + (static_cast<int64_t>(h.first_slot) * G + n) * D + lane * VEC;
    const float l = lane < h.nsplit ? pl[static_cast<int64_t>(lane) * G] : -INFINITY;
    float m = l;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
    const float w = (m == -INFINITY || l == -INFINITY) ? 0.f : expf(l - m);  // 0 for an empty part
    float sum = w;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(FULL, sum, off);
    float acc[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) acc[c] = 0.f;
    for (int j0 = 0; j0 < h.nsplit; j0 += kPartBatch) {
        float v[kPartBatch][VEC];
#pragma unroll
        for (int jj = 0; jj < kPartBatch; ++jj) {
            const int j = j0 + jj;
            if constexpr (VEC == 4) {
                const float4 x = j < h.nsplit ? *reinterpret_cast<const float4 *>(po + j * pstride)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
                v[jj][0] = x.x;
                v[jj][1] = x.y;
                v[jj][2] = x.z;
                v[jj][3] = x.w;
            } else {
#pragma unroll
                for (int c = 0; c < VEC; ++c) v[jj][c] = j < h.nsplit ? po[j * pstride + c] : 0.f;
            }
        }
#pragma unroll
        for (int jj = 0; jj < kPartBatch; ++jj) {
            const float wj = __shfl_sync(FULL, w, (j0 + jj) & 31);  // 0 past the parts
#pragma unroll
            for (int c = 0; c < VEC; ++c) acc[c] += wj * v[jj][c];
        }
    }
    const int32_t b = h.bh / Hkv, hh = h.bh - b * Hkv;
    const int64_t row = static_cast<int64_t>(b) * Hq + static_cast<int64_t>(hh) * G + n;
    const float inv = m == -INFINITY ? 0.f : 1.f / sum;
    if constexpr (VEC == 4) {
        if (out_f32) {
            *reinterpret_cast<float4 *>(out_f32 + row * D + lane * VEC) =
                make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        } else {
            *reinterpret_cast<uint2 *>(out + row * D + lane * VEC) =
                make_uint2(dev::pack_bf16(acc[0] * inv, acc[1] * inv), dev::pack_bf16(acc[2] * inv, acc[3] * inv));
        }
    } else {
#pragma unroll
        for (int c = 0; c < VEC; ++c) {
            if (out_f32)
                out_f32[row * D + lane * VEC + c] = acc[c] * inv;
            else
                out[row * D + lane * VEC + c] = __float2bfloat16_rn(acc[c] * inv);
        }
    }
    if (lane == 0) lse[row] = m == -INFINITY ? -INFINITY : m + logf(sum);
}

// Generic merge (exported as tg_lse_merge): rows with contiguous split ranges.
__global__ void lse_merge_kernel(int64_t n_rows, int32_t D, const int64_t *off, const float *po,
                                 const float *pl, __nv_bfloat16 *out, float *lse) {
    const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (r >= n_rows) return;
    const int64_t j0 = off[r], j1 = off[r + 1];
    float mx = -INFINITY;
    for (int64_t j = j0; j < j1; ++j) mx = fmaxf(mx, pl[j]);
    if (mx == -INFINITY) {
        for (int d = lane; d < D; d += 32) out[r * D + d] = __float2bfloat16_rn(0.f);
        if (lane == 0) lse[r] = -INFINITY;
        return;
    }
    float sum = 0.f;
    for (int64_t j = j0; j < j1; ++j) sum += expf(pl[j] - mx);
    const float tot = mx + logf(sum);
    for (int d = lane; d < D; d += 32) {
        float acc = 0.f;
        for (int64_t j = j0; j < j1; ++j) acc += expf(pl[j] - tot) * po[j * D + d];
        out[r * D + d] = __float2bfloat16_rn(acc);
    }
    if (lane == 0) lse[r] = tot;
}

// ------------------------------------------------------------------------------------------
// INT8 quantiser: one warp per row of D bf16 values.
// ------------------------------------------------------------------------------------------
template <int D>
__global__ void quantize_kernel(int64_t n_rows, const __nv_bfloat16 *src, int8_t *codes,
                                float *scale) {
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < n_rows; r += warps) {
        float x[PER];
        float amax = 0.f;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            x[k] = __bfloat162float(src[r * D + lane * PER + k]);
            amax = fmaxf(amax, fabsf(x[k]));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const float sc = __fdiv_rn(amax, 127.f);
        int8_t c[PER];
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            int v = 0;
            if (amax != 0.f) v = max(-127, min(127, __float2int_rn(__fdiv_rn(x[k], sc))));
            c[k] = static_cast<int8_t>(v);
        }
#pragma unroll
        for (int k = 0; k < PER; ++k) codes[r * D + lane * PER + k] = c[k];
        if (lane == 0) scale[r] = sc;
    }
}

// INT4 quantiser: one warp per row; scale = amax / 7, code = clamp(rint(x / scale), -7, 7)
// (fp32 quotient, ties to even); byte i of the packed row = (code_i + 8) | (code_{i+D/2} + 8) << 4.
template <int D>
__global__ void quantize4_kernel(int64_t n_rows, const __nv_bfloat16 *src, uint8_t *packed,
                                 float *scale) {
    constexpr int PB = D / 64;  // packed bytes per lane
    const int lane = threadIdx.x & 31;
    const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < n_rows; r += warps) {
        float lo[PB], hi[PB];
        float amax = 0.f;
#pragma unroll
        for (int k = 0; k < PB; ++k) {
            lo[k] = __bfloat162float(src[r * D + lane * PB + k]);
            hi[k] = __bfloat162float(src[r * D + D / 2 + lane * PB + k]);
            amax = fmaxf(amax, fmaxf(fabsf(lo[k]), fabsf(hi[k])));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const float sc = __fdiv_rn(amax, 7.f);
#pragma unroll
        for (int k = 0; k < PB; ++k) {
            int cl = 0, ch = 0;
            if (amax != 0.f) {
                cl = max(-7, min(7, __float2int_rn(__fdiv_rn(lo[k], sc))));
                ch = max(-7, min(7, __float2int_rn(__fdiv_rn(hi[k], sc))));
            }
            packed[r * (D / 2) + lane * PB + k] = static_cast<uint8_t>((cl + 8) | ((ch + 8) << 4));
        }
        if (lane == 0) scale[r] = sc;
    }
}

// ------------------------------------------------------------------------------------------
// Host: tensor maps, plan device state, launchers
// ------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// Tensor map over a pool of pages [rows = pages * 16][inner] with swizzled boxes of box_inner
// elements x 16 rows (128-byte swizzle, or 64-byte for the 64-byte rows of INT4 pages).
static int make_pool_map(CUtensorMap *tm, const void *base, CUtensorMapDataType dt, int elem,
                         uint64_t inner, uint64_t rows, uint32_t box_inner,
                         CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        set_cuda_error("cuTensorMapEncodeTiled unavailable", 0);
        return TG_ECUDA;
    }
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * static_cast<uint64_t>(elem)};
    cuuint32_t box[2] = {box_inner, 16};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_cuda_msg, sizeof(g_cuda_msg), "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
        return TG_ECUDA;
    }
    return TG_OK;
}

int device_num_sms(int device, int *num_sms) {
    int dev = device;
    if (dev < 0) TG_CUDA_TRY(cudaGetDevice(&dev));
    TG_CUDA_TRY(cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev));
    return TG_OK;
}

static constexpr int kSmemBudget = 232448;  // 227 KB opt-in dynamic shared memory per CTA

template <int D, bool TIERED, int NPAIRS, int SB = 8>
static int set_smem_attr(int bytes) {
    TG_CUDA_TRY(cudaFuncSetAttribute(decode_kernel<D, TIERED, NPAIRS, SB>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
    return TG_OK;
}

int device_init_plan(tg_plan *p) {
    const tg_shape &s = p->shape;
    int cur = 0;
    TG_CUDA_TRY(cudaGetDevice(&cur));
    if (p->device < 0) p->device = cur;
    if (p->device != cur) TG_CUDA_TRY(cudaSetDevice(p->device));

    // Stage geometry.
    const int KB = 16 * s.D * 2;
    const int QB = ((p->G * s.D * 2) + 1023) / 1024 * 1024;
    p->stage_bytes = 2 * KB + QB;
    const int per_stage_extra = static_cast<int>(sizeof(StageHdr)) + 16;  // header + 2 barriers
    const int np = p->pairs;
    int stages = (kSmemBudget - 1024 - np * 8) / (np * (p->stage_bytes + per_stage_extra));
    stages = stages > 8 ? 8 : stages;
    if (stages < 3) {  // a page pair plus one page in flight
        if (p->device != cur) cudaSetDevice(cur);
        return TG_EUNSUPPORTED;
    }
    p->stages = stages;
    p->smem_bytes = 1024 + np * stages * (p->stage_bytes + per_stage_extra) + np * 8;

    int rc = TG_OK;
    if (s.D == 128 && !p->tiered) rc = set_smem_attr<128, false, kPairs>(p->smem_bytes);
    else if (s.D == 128 && p->tiered && p->slow_bits == 4) rc = set_smem_attr<128, true, kPairsTiered, 4>(p->smem_bytes);
    else if (s.D == 128 && p->tiered) rc = set_smem_attr<128, true, kPairsTiered>(p->smem_bytes);
    else if (s.D == 64 && !p->tiered) rc = set_smem_attr<64, false, kPairs>(p->smem_bytes);
    else rc = TG_EUNSUPPORTED;
    if (rc == TG_OK && !p->cunits.empty()) {
        cudaError_t ce = s.D == 128
            ? cudaFuncSetAttribute(cascade_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   cascade_smem_bytes<128>())
            : cudaFuncSetAttribute(cascade_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   cascade_smem_bytes<64>());
        if (ce != cudaSuccess) {
            set_cuda_error("cudaFuncSetAttribute(cascade_kernel)", static_cast<int>(ce));
            rc = TG_ECUDA;
        }
    }
    if (rc != TG_OK) {
        if (p->device != cur) cudaSetDevice(cur);
        return rc;
    }

    // One device allocation for the plan.
    auto al = [](int64_t x) { return (x + 255) / 256 * 256; };
    const int64_t n_items = static_cast<int64_t>(p->items.size());
    const int64_t b_items = al(n_items * static_cast<int64_t>(sizeof(Item)));
    const int64_t b_woff = al((p->n_workers + 1) * 4LL);
    const int64_t b_merge = al(static_cast<int64_t>(p->merge.size()) * static_cast<int64_t>(sizeof(MergeHead)));
    const int64_t b_goff = al((p->n_groups + 1) * 8LL);
    const int64_t b_po = al(p->n_partials * p->G * s.D * 4LL);
    const int64_t b_pl = al(p->n_partials * p->G * 4LL);
    const int64_t b_emp = al(static_cast<int64_t>(p->empties.size()) * 4LL);
    const int64_t b_err = 256;  // error word + dynamic ticket counters
    const int64_t b_cu = al(static_cast<int64_t>(p->cunits.size()) * static_cast<int64_t>(sizeof(CascadeUnit)));
    const int64_t b_plan = p->lean ? al(static_cast<int64_t>(p->planned_kv.size()) * 4LL) : 0;
    p->dev_bytes = b_items + b_woff + b_merge + b_goff + b_po + b_pl + b_emp + b_err + b_cu + b_plan;
    cudaError_t e = cudaMalloc(&p->dev_base, static_cast<size_t>(p->dev_bytes));
    if (e != cudaSuccess) {
        set_cuda_error("cudaMalloc(plan)", static_cast<int>(e));
        p->dev_base = nullptr;
        if (p->device != cur) cudaSetDevice(cur);
        return TG_ENOMEM;
    }
    char *base = static_cast<char *>(p->dev_base);
    p->d_items = reinterpret_cast<Item *>(base);
    base += b_items;
    p->d_worker_off = reinterpret_cast<int32_t *>(base);
    base += b_woff;
    p->d_merge = reinterpret_cast<MergeHead *>(base);
    base += b_merge;
    p->d_group_off = reinterpret_cast<int64_t *>(base);
    base += b_goff;
    p->d_part_o = reinterpret_cast<float *>(base);
    base += b_po;
    p->d_part_lse = reinterpret_cast<float *>(base);
    base += b_pl;
    p->d_empties = reinterpret_cast<int32_t *>(base);
    base += b_emp;
    p->d_err = reinterpret_cast<uint32_t *>(base);
    p->d_dyn = p->d_err + 16;
    base += b_err;
    p->d_cunits = p->cunits.empty() ? nullptr : reinterpret_cast<CascadeUnit *>(base);
    base += b_cu;
    p->d_planned = p->lean ? reinterpret_cast<int32_t *>(base) : nullptr;

    rc = TG_OK;
    auto up = [&](void *dst, const void *src, int64_t bytes) {
        if (bytes <= 0 || rc != TG_OK) return;
        cudaError_t ee = cudaMemcpy(dst, src, static_cast<size_t>(bytes), cudaMemcpyHostToDevice);
        if (ee != cudaSuccess) {
            set_cuda_error("cudaMemcpy(plan)", static_cast<int>(ee));
            rc = TG_ECUDA;
        }
    };
    up(p->d_cunits, p->cunits.data(), static_cast<int64_t>(p->cunits.size()) * static_cast<int64_t>(sizeof(CascadeUnit)));
    up(p->d_items, p->items.data(), n_items * static_cast<int64_t>(sizeof(Item)));
    up(p->d_worker_off, p->worker_off.data(), (p->n_workers + 1) * 4LL);
    up(p->d_merge, p->merge.data(), static_cast<int64_t>(p->merge.size()) * static_cast<int64_t>(sizeof(MergeHead)));
    up(p->d_group_off, p->group_off.data(), (p->n_groups + 1) * 8LL);
    up(p->d_empties, p->empties.data(), static_cast<int64_t>(p->empties.size()) * 4LL);
    if (p->lean) up(p->d_planned, p->planned_kv.data(), static_cast<int64_t>(p->planned_kv.size()) * 4LL);
    if (rc == TG_OK) {
        cudaError_t ee = cudaMemset(p->d_err, 0, 256);
        if (ee != cudaSuccess) { set_cuda_error("cudaMemset(plan)", static_cast<int>(ee)); rc = TG_ECUDA; }
    }
    if (p->device != cur) cudaSetDevice(cur);
    return rc;
}

static void timing_free(tg_plan *p) {
    for (void *e : p->tev) cudaEventDestroy(static_cast<cudaEvent_t>(e));
    p->tev.clear();
    p->tev_cap = 0;
    p->tev_count = 0;
}

void device_free_plan(tg_plan *p) {
    timing_free(p);
    if (p->d_trace) {
        cudaFree(p->d_trace);
        p->d_trace = nullptr;
    }
    if (p->dev_base) {
        int cur = 0;
        cudaGetDevice(&cur);
        if (p->device >= 0 && p->device != cur) cudaSetDevice(p->device);
        cudaFree(p->dev_base);
        if (p->device >= 0 && p->device != cur) cudaSetDevice(cur);
        p->dev_base = nullptr;
    }
}

static bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

static int get_map(tg_plan *p, int idx, const void *base, CUtensorMapDataType dt, int elem,
                   uint64_t pages, uint32_t box_inner, bool int4 = false) {
    if (p->tm_key[idx] == base) return TG_OK;
    int rc = make_pool_map(reinterpret_cast<CUtensorMap *>(p->tmaps[idx]), base, dt, elem,
                           static_cast<uint64_t>(int4 ? p->shape.D / 2 : p->shape.D), pages * 16, box_inner,
                           int4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc == TG_OK) p->tm_key[idx] = base;
    return rc;
}

static int check_device(const tg_plan *p) {
    int cur = 0;
    TG_CUDA_TRY(cudaGetDevice(&cur));
    return cur == p->device ? TG_OK : TG_EINVAL;
}

// Timing hook: event k (0 = before the decode kernel, 1 = after it, 2 = after the merge
// kernel) of this call. A recorded call loses the launch overlap of the merge kernel.
static void timing_mark(tg_plan *p, int k, cudaStream_t stream) {
    if (p->tev_count >= p->tev_cap) return;
    cudaEventRecord(static_cast<cudaEvent_t>(p->tev[3 * p->tev_count + k]), stream);
    if (k == 2) ++p->tev_count;
}

// Decode kernel launch, as a programmatic dependent of whatever precedes it in the stream.
typedef void (*DecodeFn)(DecodeArgs, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap);
static int launch_decode(tg_plan *p, DecodeFn fn, const DecodeArgs &a, const CUtensorMap &m0,
                         const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3,
                         cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p->grid));
    cfg.blockDim = dim3(static_cast<unsigned>(p->pairs * 64));
    cfg.dynamicSmemBytes = static_cast<size_t>(p->smem_bytes);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, fn, a, m0, m1, m2, m3));
    return TG_OK;
}

// Merge kernel of the split heads (optionally a programmatic dependent launch), by the most parts
// a head of the plan has: up to 8 (merge_warps == 1), one warp per query row, 8 rows per CTA,
// its parts loaded 4 at a time; 9 to kLaneParts (merge_warps <= 4), one warp per query row with
// a lane per part (fewer dependent rounds for these heads; measured: config 2 103.8 -> 102.0
// us, while heads of 3 parts ran slower this way, 83 -> 93 us on config 4, the kernel holding
// twice the registers); more, one CTA per row, its warps splitting the head's parts.
static int launch_merge(const tg_plan *p, const MergeHead *d_merge, const float *po, const float *pl,
                        void *out, float *lse, cudaStream_t stream, bool pdl) {
    constexpr int kRowsPerCta = 8;
    static_assert(kLaneParts == 4 * 8, "lane merge: merge_warps <= 4 means at most 32 parts");
    const int64_t n_rows = static_cast<int64_t>(p->merge.size()) * p->G;
    const bool rows = p->merge_warps == 1;
    const bool lanes = !rows && p->merge_warps <= 4;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(rows || lanes ? (n_rows + kRowsPerCta - 1) / kRowsPerCta : n_rows));
    cfg.blockDim = dim3(static_cast<unsigned>(rows || lanes ? 32 * kRowsPerCta : 32 * p->merge_warps));
    cfg.dynamicSmemBytes = !rows && !lanes ? static_cast<size_t>(p->merge_warps) * (2 + p->shape.D) * 4 : 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    const int32_t G = p->G, Hq = p->shape.Hq, Hkv = p->shape.Hkv;
    __nv_bfloat16 *o = p->out_f32 ? nullptr : static_cast<__nv_bfloat16 *>(out);
    float *of = p->out_f32 ? static_cast<float *>(out) : nullptr;
    if (p->shape.D == 128) {
        if (rows) TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, split_merge_kernel<128, true>, d_merge, n_rows, G, Hq, Hkv, po, pl, o, of, lse));
        else if (lanes) TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, lane_merge_kernel<128>, d_merge, n_rows, G, Hq, Hkv, po, pl, o, of, lse));
        else TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, split_merge_kernel<128, false>, d_merge, n_rows, G, Hq, Hkv, po, pl, o, of, lse));
    } else {
        if (rows) TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, split_merge_kernel<64, true>, d_merge, n_rows, G, Hq, Hkv, po, pl, o, of, lse));
        else if (lanes) TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, lane_merge_kernel<64>, d_merge, n_rows, G, Hq, Hkv, po, pl, o, of, lse));
        else TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, split_merge_kernel<64, false>, d_merge, n_rows, G, Hq, Hkv, po, pl, o, of, lse));
    }
    return TG_OK;
}

// Merge kernel of the split heads, as a programmatic dependent launch of the decode kernel;
// then close the call's timing record.
static int finish_call(tg_plan *p, void *out, float *lse, cudaStream_t stream) {
    timing_mark(p, 1, stream);
    if (!p->merge.empty()) {
        const int rc = launch_merge(p, p->d_merge, p->d_part_o, p->d_part_lse, out, lse, stream, true);
        if (rc != TG_OK) return rc;
    }
    timing_mark(p, 2, stream);
    return TG_OK;
}

// Lean kernel launch (whole-head plans of short heads), as a programmatic dependent of whatever
// precedes it in the stream.
template <int D, int G>
static int launch_lean_t(const tg_plan *p, const LeanArgs &a, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(static_cast<int64_t>(p->shape.B) * p->shape.Hkv));
    cfg.blockDim = dim3(kLeanWarps * 32);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, lean_decode_kernel<D, G>, a));
    return TG_OK;
}

static int launch_lean(const tg_plan *p, const void *q, const void *k_pages, const void *v_pages,
                       const int32_t *page_table, const int64_t *head_page_off,
                       const int32_t *head_kv_len, const int32_t *group_of_head, float scale,
                       void *out, float *lse, cudaStream_t stream) {
    LeanArgs a{};
    a.Hq = p->shape.Hq;
    a.Hkv = p->shape.Hkv;
    a.scale_log2 = scale * 1.44269504088896340736f;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.k_pages = static_cast<const __nv_bfloat16 *>(k_pages);
    a.v_pages = static_cast<const __nv_bfloat16 *>(v_pages);
    a.table = page_table;
    a.head_off = head_page_off;
    a.group_of_head = group_of_head;
    a.group_off = p->d_group_off;
    a.n_groups = p->n_groups;
    a.kv_len_dev = head_kv_len;
    a.planned = p->d_planned;
    a.num_pages = p->shape.num_pages;
    a.out = p->out_f32 ? nullptr : static_cast<__nv_bfloat16 *>(out);
    a.out_f32 = p->out_f32 ? static_cast<float *>(out) : nullptr;
    a.lse = lse;
    a.err = p->d_err;
    a.early_prologue = p->early_prologue ? 1 : 0;
    const int G = p->G;
    if (p->shape.D == 128) {
        if (G == 1) return launch_lean_t<128, 1>(p, a, stream);
        if (G == 2) return launch_lean_t<128, 2>(p, a, stream);
        if (G == 4) return launch_lean_t<128, 4>(p, a, stream);
        return launch_lean_t<128, 8>(p, a, stream);
    }
    if (G == 1) return launch_lean_t<64, 1>(p, a, stream);
    if (G == 2) return launch_lean_t<64, 2>(p, a, stream);
    if (G == 4) return launch_lean_t<64, 4>(p, a, stream);
    return launch_lean_t<64, 8>(p, a, stream);
}

static DecodeArgs base_args(const tg_plan *p, const void *q, const int32_t *kv, float scale,
                            void *out, float *lse) {
    DecodeArgs a{};
    a.items = p->d_items;
    a.worker_off = p->d_worker_off;
    a.n_workers = p->n_workers;
    a.B = p->shape.B;
    a.Hq = p->shape.Hq;
    a.Hkv = p->shape.Hkv;
    a.G = p->G;
    a.stages = p->stages;
    a.stage_bytes = p->stage_bytes;
    a.scale_log2 = scale * 1.44269504088896340736f;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.group_off = p->d_group_off;
    a.n_groups = p->n_groups;
    a.kv_len_dev = kv;
    a.num_pages = p->shape.num_pages;
    a.num_slow_pages = p->shape.num_slow_pages;
    a.out = p->out_f32 ? nullptr : static_cast<__nv_bfloat16 *>(out);
    a.out_f32 = p->out_f32 ? static_cast<float *>(out) : nullptr;
    a.lse = lse;
    a.part_o = p->d_part_o;
    a.part_lse = p->d_part_lse;
    a.empties = p->d_empties;
    a.n_empty = static_cast<int32_t>(p->empties.size());
    a.err = p->d_err;
    a.trace = p->d_trace;
    a.dyn_first = p->dyn_first;
    a.n_dyn = p->n_dyn;
    a.dyn_next = p->d_dyn;
    a.early_prologue = p->early_prologue ? 1 : 0;
    a.wait_ns = p->wait_ns;
    a.withhold = p->withhold;
    a.capacity = p->capacity ? 1 : 0;
    return a;
}

}  // namespace tg

// ------------------------------------------------------------------------------------------
// ABI entry points (device)
// ------------------------------------------------------------------------------------------
using namespace tg;

extern "C" const char *tg_last_cuda_error(void) { return g_cuda_msg; }

static int decode_bf16(tg_plan *p, const void *q, const void *k_pages, const void *v_pages,
                       const int32_t *page_table, const int64_t *head_page_off,
                       const int32_t *head_kv_len, const int32_t *group_of_head, float scale,
                       void *out, float *lse, float *token_scores, tg_stream stream_) {
    if (!p || p->host_only || p->tiered) return TG_EINVAL;
    if (!q || !out || !lse || !head_kv_len || !aligned16(q) || !aligned16(out) || !aligned16(lse))
        return TG_EINVAL;
    const bool any_items = !p->items.empty();
    const bool launch = p->grid > 0;
    if (any_items && (!k_pages || !v_pages || !page_table || !head_page_off || !group_of_head ||
                      !aligned16(k_pages) || !aligned16(v_pages) || p->shape.num_pages < 1))
        return TG_EINVAL;
    int rc = check_device(p);
    if (rc != TG_OK) return rc;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    const bool cascade = !p->cunits.empty();
    if (cascade && (!k_pages || !v_pages || !page_table || !head_page_off ||
                    !aligned16(k_pages) || !aligned16(v_pages) || p->shape.num_pages < 1))
        return TG_EINVAL;
    if (p->lean && !token_scores) {
        // Whole-head plan of short heads: the lean kernel, one CTA per (sequence, KV head).
        const int64_t heads = static_cast<int64_t>(p->shape.B) * p->shape.Hkv;
        timing_mark(p, 0, stream);
        if (heads > 0) {
            if (!k_pages || !v_pages || !page_table || !head_page_off || !aligned16(k_pages) ||
                !aligned16(v_pages))
                return TG_EINVAL;
            rc = launch_lean(p, q, k_pages, v_pages, page_table, head_page_off, head_kv_len,
                             group_of_head, scale, out, lse, stream);
            if (rc != TG_OK) return rc;
        }
        return finish_call(p, out, lse, stream);
    }
    if (cascade) {
        // Shared runs first (the decode kernel that follows waits for them before it starts).
        rc = get_map(p, 0, k_pages, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p->shape.num_pages, 64);
        if (rc == TG_OK) rc = get_map(p, 1, v_pages, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p->shape.num_pages, 64);
        if (rc != TG_OK) return rc;
        CascadeArgs c{};
        c.units = p->d_cunits;
        c.G = p->G;
        c.Hq = p->shape.Hq;
        c.Hkv = p->shape.Hkv;
        c.scale_log2 = scale * 1.44269504088896340736f;
        c.q = static_cast<const __nv_bfloat16 *>(q);
        c.table = page_table;
        c.head_off = head_page_off;
        c.kv_len_dev = head_kv_len;
        c.num_pages = p->shape.num_pages;
        c.part_o = p->d_part_o;
        c.part_lse = p->d_part_lse;
        c.err = p->d_err;
        c.wait_ns = p->wait_ns;
        timing_mark(p, 0, stream);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(p->cunits.size()));
        cfg.blockDim = dim3(kTcThreads);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const CUtensorMap &tk = *reinterpret_cast<const CUtensorMap *>(p->tmaps[0]);
        const CUtensorMap &tv = *reinterpret_cast<const CUtensorMap *>(p->tmaps[1]);
        if (p->shape.D == 128) {
            cfg.dynamicSmemBytes = cascade_smem_bytes<128>();
            TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, cascade_kernel<128>, c, tk, tv));
        } else {
            cfg.dynamicSmemBytes = cascade_smem_bytes<64>();
            TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, cascade_kernel<64>, c, tk, tv));
        }
    }
    if (launch) {
        if (any_items) rc = get_map(p, 0, k_pages, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p->shape.num_pages, 64);
        if (rc == TG_OK && any_items) rc = get_map(p, 1, v_pages, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p->shape.num_pages, 64);
        if (rc != TG_OK) return rc;
        DecodeArgs a = base_args(p, q, head_kv_len, scale, out, lse);
        if (!cascade) timing_mark(p, 0, stream);
        a.table = page_table;
        a.head_off = head_page_off;
        a.group_of_head = group_of_head;
        a.token_scores = token_scores;
        // The cascade kernel before this one waited for the previous step's merge before it let
        // this grid launch, and writes other partial slots: the decode overlaps it and waits for
        // it only before exiting (so the merge that follows sees both).
        a.late_wait = cascade ? 1 : 0;
        const CUtensorMap &tk = *reinterpret_cast<const CUtensorMap *>(p->tmaps[0]);
        const CUtensorMap &tv = *reinterpret_cast<const CUtensorMap *>(p->tmaps[1]);
        if (p->shape.D == 128)
            rc = launch_decode(p, decode_kernel<128, false, kPairs>, a, tk, tv, tk, tv, stream);
        else
            rc = launch_decode(p, decode_kernel<64, false, kPairs>, a, tk, tv, tk, tv, stream);
        if (rc != TG_OK) return rc;
    } else if (!cascade) {
        timing_mark(p, 0, stream);
    }
    return finish_call(p, out, lse, stream);
}

extern "C" int tg_ragged_paged_decode(tg_plan *p, const void *q, const void *k_pages,
                                      const void *v_pages, const int32_t *page_table,
                                      const int64_t *head_page_off, const int32_t *head_kv_len,
                                      const int32_t *group_of_head, float scale, void *out,
                                      float *lse, tg_stream stream) {
    return decode_bf16(p, q, k_pages, v_pages, page_table, head_page_off, head_kv_len,
                       group_of_head, scale, out, lse, nullptr, stream);
}

extern "C" int tg_ragged_paged_decode_scores(tg_plan *p, const void *q, const void *k_pages,
                                             const void *v_pages, const int32_t *page_table,
                                             const int64_t *head_page_off,
                                             const int32_t *head_kv_len,
                                             const int32_t *group_of_head, float scale,
                                             void *out, float *lse, float *token_scores,
                                             tg_stream stream) {
    if (!token_scores || (reinterpret_cast<uintptr_t>(token_scores) & 3u)) return TG_EINVAL;
    return decode_bf16(p, q, k_pages, v_pages, page_table, head_page_off, head_kv_len,
                       group_of_head, scale, out, lse, token_scores, stream);
}

extern "C" int tg_tiered_decode(tg_plan *p, const void *q, const int8_t *k_q8,
                                const int8_t *v_q8, const float *k_scale, const float *v_scale,
                                const int32_t *slow_page_table, const int64_t *slow_head_off,
                                const void *k_fast, const void *v_fast,
                                const int32_t *fast_page_table, const int64_t *fast_head_off,
                                const int32_t *head_kv_len, const int32_t *head_fast_len,
                                float scale, void *out, float *lse, tg_stream stream_) {
    if (!p || p->host_only || !p->tiered) return TG_EINVAL;
    if (!q || !out || !lse || !head_kv_len || !head_fast_len || !aligned16(q) || !aligned16(out) ||
        !aligned16(lse))
        return TG_EINVAL;
    bool has_slow = false, has_fast = false;
    for (const Item &it : p->items) (it.flags & kItemSlow ? has_slow : has_fast) = true;
    if (has_slow && (!k_q8 || !v_q8 || !k_scale || !v_scale || !slow_page_table || !slow_head_off ||
                     !aligned16(k_q8) || !aligned16(v_q8) || !aligned16(k_scale) ||
                     !aligned16(v_scale) || p->shape.num_slow_pages < 1))
        return TG_EINVAL;
    if (has_fast && (!k_fast || !v_fast || !fast_page_table || !fast_head_off ||
                     !aligned16(k_fast) || !aligned16(v_fast) || p->shape.num_pages < 1))
        return TG_EINVAL;
    int rc = check_device(p);
    if (rc != TG_OK) return rc;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (p->grid > 0) {
        if (has_fast) {
            rc = get_map(p, 0, k_fast, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p->shape.num_pages, 64);
            if (rc == TG_OK) rc = get_map(p, 1, v_fast, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p->shape.num_pages, 64);
        }
        if (rc == TG_OK && has_slow) {
            const bool i4 = p->slow_bits == 4;
            const uint32_t box = i4 ? static_cast<uint32_t>(p->shape.D / 2) : 128u;
            rc = get_map(p, 2, k_q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p->shape.num_slow_pages, box, i4);
            if (rc == TG_OK) rc = get_map(p, 3, v_q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p->shape.num_slow_pages, box, i4);
        }
        if (rc != TG_OK) return rc;
        DecodeArgs a = base_args(p, q, head_kv_len, scale, out, lse);
        timing_mark(p, 0, stream);
        a.table = fast_page_table;
        a.head_off = fast_head_off;
        a.group_of_head = nullptr;
        a.slow_table = slow_page_table;
        a.slow_off = slow_head_off;
        a.slow_table_len = p->slow_table_len;
        a.k_scale = k_scale;
        a.v_scale = v_scale;
        a.fast_len_dev = head_fast_len;
        // The fast tier's rows are bounded by its whole table [group_off[0], group_off[n]).
        const CUtensorMap *maps = reinterpret_cast<const CUtensorMap *>(p->tmaps[0]);
        if (p->slow_bits == 4)
            rc = launch_decode(p, decode_kernel<128, true, kPairsTiered, 4>, a, maps[has_fast ? 0 : 2],
                               maps[has_fast ? 1 : 3], maps[has_slow ? 2 : 0], maps[has_slow ? 3 : 1], stream);
        else
            rc = launch_decode(p, decode_kernel<128, true, kPairsTiered>, a, maps[has_fast ? 0 : 2],
                               maps[has_fast ? 1 : 3], maps[has_slow ? 2 : 0], maps[has_slow ? 3 : 1], stream);
        if (rc != TG_OK) return rc;
    } else {
        timing_mark(p, 0, stream);
    }
    return finish_call(p, out, lse, stream);
}

extern "C" int tg_plan_status(tg_plan *p, tg_stream stream_) {
    if (!p || p->host_only) return TG_EINVAL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    uint32_t err = 0;
    TG_CUDA_TRY(cudaMemcpyAsync(&err, p->d_err, 4, cudaMemcpyDeviceToHost, stream));
    TG_CUDA_TRY(cudaStreamSynchronize(stream));
    TG_CUDA_TRY(cudaMemsetAsync(p->d_err, 0, 4, stream));
    // A timed-out call may leave the dynamic ticket part-counted: reset it.
    if (err & kErrTimeout) TG_CUDA_TRY(cudaMemsetAsync(p->d_dyn, 0, 8, stream));
    TG_CUDA_TRY(cudaStreamSynchronize(stream));
    if (err & kErrTimeout) return TG_ETIMEOUT;
    if (err & (kErrBadPage | kErrBadRow | kErrPlan)) return TG_EBADPAGE;
    return TG_OK;
}

extern "C" int tg_lse_merge(int64_t n_rows, int32_t D, const int64_t *row_split_off,
                            const float *part_o, const float *part_lse, void *out, float *lse,
                            tg_stream stream_) {
    if (n_rows < 0 || D < 1 || D > 4096) return TG_EINVAL;
    if (n_rows == 0) return TG_OK;
    if (!row_split_off || !out || !lse) return TG_EINVAL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    const int threads = 256;
    const int64_t blocks = (n_rows * 32 + threads - 1) / threads;
    lse_merge_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
        n_rows, D, row_split_off, part_o, part_lse, static_cast<__nv_bfloat16 *>(out), lse);
    TG_CUDA_TRY(cudaGetLastError());
    return TG_OK;
}

extern "C" int tg_quantize_int8(int64_t n_rows, int32_t D, const void *src, int8_t *codes,
                                float *scale, tg_stream stream_) {
    if (n_rows < 0 || (D != 64 && D != 128)) return n_rows < 0 ? TG_EINVAL : TG_EUNSUPPORTED;
    if (n_rows == 0) return TG_OK;
    if (!src || !codes || !scale) return TG_EINVAL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int threads = 256;
    int64_t blocks = (n_rows * 32 + threads - 1) / threads;
    if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
    if (D == 128)
        quantize_kernel<128><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
            n_rows, static_cast<const __nv_bfloat16 *>(src), codes, scale);
    else
        quantize_kernel<64><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
            n_rows, static_cast<const __nv_bfloat16 *>(src), codes, scale);
    TG_CUDA_TRY(cudaGetLastError());
    return TG_OK;
}

extern "C" int tg_quantize_int4(int64_t n_rows, int32_t D, const void *src, uint8_t *packed,
                                float *scale, tg_stream stream_) {
    if (n_rows < 0 || (D != 64 && D != 128)) return n_rows < 0 ? TG_EINVAL : TG_EUNSUPPORTED;
    if (n_rows == 0) return TG_OK;
    if (!src || !packed || !scale) return TG_EINVAL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int threads = 256;
    int64_t blocks = (n_rows * 32 + threads - 1) / threads;
    if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
    if (D == 128)
        quantize4_kernel<128><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
            n_rows, static_cast<const __nv_bfloat16 *>(src), packed, scale);
    else
        quantize4_kernel<64><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
            n_rows, static_cast<const __nv_bfloat16 *>(src), packed, scale);
    TG_CUDA_TRY(cudaGetLastError());
    return TG_OK;
}

extern "C" int tg_plan_timing_enable(tg_plan *p, int32_t max_calls) {
    if (!p || p->host_only || max_calls < 0) return TG_EINVAL;
    timing_free(p);
    if (max_calls == 0) return TG_OK;
    p->tev.assign(static_cast<size_t>(max_calls) * 3, nullptr);
    for (auto &e : p->tev) {
        cudaEvent_t ev;
        cudaError_t r = cudaEventCreate(&ev);
        if (r != cudaSuccess) {
            set_cuda_error("cudaEventCreate", static_cast<int>(r));
            for (void *x : p->tev)
                if (x) cudaEventDestroy(static_cast<cudaEvent_t>(x));
            p->tev.clear();
            return TG_ECUDA;
        }
        e = ev;
    }
    p->tev_cap = max_calls;
    p->tev_count = 0;
    return TG_OK;
}

extern "C" int tg_plan_timing_read(tg_plan *p, int32_t *n_calls, double *decode_ms,
                                   double *merge_ms) {
    if (!p || !n_calls || !decode_ms || !merge_ms) return TG_EINVAL;
    *n_calls = p->tev_count;
    *decode_ms = 0.0;
    *merge_ms = 0.0;
    if (p->tev_count == 0) return TG_OK;
    TG_CUDA_TRY(cudaEventSynchronize(static_cast<cudaEvent_t>(p->tev[3 * p->tev_count - 1])));
    for (int32_t i = 0; i < p->tev_count; ++i) {
        float a = 0.f, b = 0.f;
        TG_CUDA_TRY(cudaEventElapsedTime(&a, static_cast<cudaEvent_t>(p->tev[3 * i]),
                                         static_cast<cudaEvent_t>(p->tev[3 * i + 1])));
        TG_CUDA_TRY(cudaEventElapsedTime(&b, static_cast<cudaEvent_t>(p->tev[3 * i + 1]),
                                         static_cast<cudaEvent_t>(p->tev[3 * i + 2])));
        *decode_ms += a;
        *merge_ms += b;
    }
    p->tev_count = 0;
    return TG_OK;
}

extern "C" int tg_plan_trace_enable(tg_plan *p, int32_t on) {
    if (!p || p->host_only) return TG_EINVAL;
    if (p->d_trace) {
        cudaFree(p->d_trace);
        p->d_trace = nullptr;
    }
    if (!on || p->n_workers == 0) return TG_OK;
    const size_t bytes = static_cast<size_t>(p->n_workers) * kTraceWords * sizeof(uint64_t);
    cudaError_t e = cudaMalloc(&p->d_trace, bytes);
    if (e != cudaSuccess) {
        set_cuda_error("cudaMalloc(trace)", static_cast<int>(e));
        p->d_trace = nullptr;
        return TG_ENOMEM;
    }
    TG_CUDA_TRY(cudaMemset(p->d_trace, 0, bytes));
    return TG_OK;
}

extern "C" int tg_plan_trace_read(tg_plan *p, uint64_t *trace, tg_stream stream_) {
    if (!p || !trace || !p->d_trace) return TG_EINVAL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    TG_CUDA_TRY(cudaMemcpyAsync(trace, p->d_trace, static_cast<size_t>(p->n_workers) * kTraceWords * 8,
                                cudaMemcpyDeviceToHost, stream));
    TG_CUDA_TRY(cudaStreamSynchronize(stream));
    return TG_OK;
}

// ------------------------------------------------------------------------------------------
// Decode without device allocation.
//
// For callers that must not allocate device memory after start-up (an engine that reserves
// the whole device for its KV pool and treats any later cudaMalloc as a failure, a plug-in
// whose host framework owns every device allocation, a runtime that allows allocation only
// during initialisation). Their scratch lives in one file-scope device array of fixed size;
// every GPU that loads this library holds it until the process exits. The host code below
// never names the array as a device address: it asks the runtime for the array's device
// address once per device and passes that address to the kernels.
// ------------------------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kNoAllocMaxDevices] = {};

// One-time set-up on the current device: the array's device address, a cleared error word,
// and the decode kernels' shared-memory limit.
int noalloc_setup(int dev, void **ptr) {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            set_cuda_error("cudaGetSymbolAddress(scratch)", static_cast<int>(e));
            return TG_ECUDA;
        }
        TG_CUDA_TRY(cudaMemset(p, 0, 256));
        TG_CUDA_TRY(cudaFuncSetAttribute(decode_kernel<128, false, tg::kPairs>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget));
        TG_CUDA_TRY(cudaFuncSetAttribute(decode_kernel<64, false, tg::kPairs>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget));
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return TG_OK;
}
}  // namespace

extern "C" int tg_ragged_paged_decode_noalloc(tg_plan *p, const void *q, const void *k_pages,
                                              const void *v_pages, const int32_t *page_table,
                                              const int64_t *head_page_off,
                                              const int32_t *head_kv_len,
                                              const int32_t *group_of_head, float scale,
                                              void *out, float *lse, tg_stream stream_) {
    if (!p || p->tiered) return TG_EINVAL;
    if (!p->cunits.empty()) return TG_EUNSUPPORTED;  // cascade units live in the plan's memory
    int dev = 0;
    TG_CUDA_TRY(cudaGetDevice(&dev));
    // A plan made for one device (host-only plans may name none: device -1) runs only there.
    if (p->device >= 0 && p->device != dev) return TG_EINVAL;
    if (!q || !out || !lse || !head_kv_len || !aligned16(q) || !aligned16(out) || !aligned16(lse))
        return TG_EINVAL;
    const bool any_items = !p->items.empty();
    if (any_items && (!k_pages || !v_pages || !page_table || !head_page_off || !group_of_head ||
                      !aligned16(k_pages) || !aligned16(v_pages) || p->shape.num_pages < 1))
        return TG_EINVAL;

    // Scratch layout: [0, 256) error word and dynamic tickets, then the work list, worker
    // offsets, merge list, group offsets, empty heads, partial results.
    auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t b_items = al(p->items.size() * sizeof(Item));
    const size_t b_woff = al((static_cast<size_t>(p->n_workers) + 1) * 4);
    const size_t b_merge = al(p->merge.size() * sizeof(MergeHead));
    const size_t b_goff = al((static_cast<size_t>(p->n_groups) + 1) * 8);
    const size_t b_emp = al(p->empties.size() * 4);
    const size_t b_po = al(static_cast<size_t>(p->n_partials) * p->G * p->shape.D * 4);
    const size_t b_pl = al(static_cast<size_t>(p->n_partials) * p->G * 4);
    const size_t need = 256 + b_items + b_woff + b_merge + b_goff + b_emp + b_po + b_pl;
    if (need > kNoAllocScratchBytes) {
        std::snprintf(g_cuda_msg, sizeof(g_cuda_msg),
                      "tg_ragged_paged_decode_noalloc: plan needs %zu bytes of scratch, the "
                      "fixed scratch holds %zu",
                      need, kNoAllocScratchBytes);
        return TG_ENOMEM;
    }
    // Stage geometry (as for a device plan).
    const tg_shape &s = p->shape;
    const int KB = 16 * s.D * 2;
    const int QB = ((p->G * s.D * 2) + 1023) / 1024 * 1024;
    const int stage_bytes = 2 * KB + QB;
    const int per_stage_extra = static_cast<int>(sizeof(StageHdr)) + 16;
    int stages = (kSmemBudget - 1024 - tg::kPairs * 8) / (tg::kPairs * (stage_bytes + per_stage_extra));
    stages = stages > 8 ? 8 : stages;
    if (stages < 2) return TG_EUNSUPPORTED;
    const int smem_bytes = 1024 + tg::kPairs * stages * (stage_bytes + per_stage_extra) + tg::kPairs * 8;

    if (dev < 0 || dev >= kNoAllocMaxDevices) return TG_EUNSUPPORTED;
    void *base_v = nullptr;
    int rc = noalloc_setup(dev, &base_v);
    if (rc != TG_OK) return rc;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);

    char *base = static_cast<char *>(base_v);
    uint32_t *d_err = reinterpret_cast<uint32_t *>(base);
    uint32_t *d_dyn = d_err + 16;
    char *at = base + 256;
    Item *d_items = reinterpret_cast<Item *>(at);
    at += b_items;
    int32_t *d_woff = reinterpret_cast<int32_t *>(at);
    at += b_woff;
    MergeHead *d_merge = reinterpret_cast<MergeHead *>(at);
    at += b_merge;
    int64_t *d_goff = reinterpret_cast<int64_t *>(at);
    at += b_goff;
    int32_t *d_emp = reinterpret_cast<int32_t *>(at);
    at += b_emp;
    float *d_po = reinterpret_cast<float *>(at);
    at += b_po;
    float *d_pl = reinterpret_cast<float *>(at);

    // The scratch keeps the previous call's contents: the dynamic tickets must start at zero
    // (a call that timed out leaves them part-counted); the error word collects the calls'
    // range errors and timeouts until tg_ragged_paged_decode_noalloc_status reads and clears
    // it; the work list is written afresh (plain copies, no allocation).
    TG_CUDA_TRY(cudaMemsetAsync(d_dyn, 0, 8, stream));
    if (!p->items.empty())
        TG_CUDA_TRY(cudaMemcpyAsync(d_items, p->items.data(), p->items.size() * sizeof(Item),
                                    cudaMemcpyHostToDevice, stream));
    TG_CUDA_TRY(cudaMemcpyAsync(d_woff, p->worker_off.data(), (p->worker_off.size()) * 4,
                                cudaMemcpyHostToDevice, stream));
    if (!p->merge.empty())
        TG_CUDA_TRY(cudaMemcpyAsync(d_merge, p->merge.data(), p->merge.size() * sizeof(MergeHead),
                                    cudaMemcpyHostToDevice, stream));
    TG_CUDA_TRY(cudaMemcpyAsync(d_goff, p->group_off.data(), p->group_off.size() * 8,
                                cudaMemcpyHostToDevice, stream));
    if (!p->empties.empty())
        TG_CUDA_TRY(cudaMemcpyAsync(d_emp, p->empties.data(), p->empties.size() * 4,
                                    cudaMemcpyHostToDevice, stream));

    if (p->grid > 0) {
        if (any_items) {
            rc = get_map(p, 0, k_pages, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, s.num_pages, 64);
            if (rc == TG_OK) rc = get_map(p, 1, v_pages, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, s.num_pages, 64);
            if (rc != TG_OK) return rc;
        }
        DecodeArgs a{};
        a.items = d_items;
        a.worker_off = d_woff;
        a.n_workers = p->n_workers;
        a.B = s.B;
        a.Hq = s.Hq;
        a.Hkv = s.Hkv;
        a.G = p->G;
        a.stages = stages;
        a.stage_bytes = stage_bytes;
        a.scale_log2 = scale * 1.44269504088896340736f;
        a.q = static_cast<const __nv_bfloat16 *>(q);
        a.table = page_table;
        a.head_off = head_page_off;
        a.group_of_head = group_of_head;
        a.group_off = d_goff;
        a.n_groups = p->n_groups;
        a.kv_len_dev = head_kv_len;
        a.num_pages = s.num_pages;
        a.num_slow_pages = s.num_slow_pages;
        a.out = p->out_f32 ? nullptr : static_cast<__nv_bfloat16 *>(out);
        a.out_f32 = p->out_f32 ? static_cast<float *>(out) : nullptr;
        a.lse = lse;
        a.part_o = d_po;
        a.part_lse = d_pl;
        a.empties = d_emp;
        a.n_empty = static_cast<int32_t>(p->empties.size());
        a.err = d_err;
        a.trace = nullptr;
        a.dyn_first = p->dyn_first;
        a.n_dyn = p->n_dyn;
        a.dyn_next = d_dyn;
        a.early_prologue = 0;
        a.wait_ns = p->wait_ns;
        a.withhold = p->withhold;
        const CUtensorMap &tk = *reinterpret_cast<const CUtensorMap *>(p->tmaps[0]);
        const CUtensorMap &tv = *reinterpret_cast<const CUtensorMap *>(p->tmaps[1]);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(p->grid));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
        cfg.stream = stream;
        if (s.D == 128)
            TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, decode_kernel<128, false, tg::kPairs>, a, tk, tv, tk, tv));
        else
            TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, decode_kernel<64, false, tg::kPairs>, a, tk, tv, tk, tv));
    }
    if (!p->merge.empty())
        return launch_merge(p, reinterpret_cast<const MergeHead *>(d_merge), reinterpret_cast<const float *>(d_po),
                            reinterpret_cast<const float *>(d_pl), out, lse, stream, false);
    return TG_OK;
}

extern "C" int tg_ragged_paged_decode_noalloc_status(tg_stream stream_) {
    int dev = 0;
    TG_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kNoAllocMaxDevices) return TG_EUNSUPPORTED;
    void *base = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        base = g_noalloc_ptr[dev];
    }
    if (!base) return TG_OK;  // no call has run on this device yet
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    uint32_t err = 0;
    TG_CUDA_TRY(cudaMemcpyAsync(&err, base, 4, cudaMemcpyDeviceToHost, stream));
    TG_CUDA_TRY(cudaStreamSynchronize(stream));
    TG_CUDA_TRY(cudaMemsetAsync(base, 0, 4, stream));
    TG_CUDA_TRY(cudaStreamSynchronize(stream));
    if (err & kErrTimeout) return TG_ETIMEOUT;
    if (err & (kErrBadPage | kErrBadRow | kErrPlan)) return TG_EBADPAGE;
    return TG_OK;
}
