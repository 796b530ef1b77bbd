// Decode-step write path: append one token per (sequence, KV head) into a head whose footprint
// is fixed, and the H2O score bookkeeping that chooses which retained token a full head gives up.
//
// Sources: "Tangram" explainer, 三大机制 1 (Budget Reservation: a head's post-compression
// footprint is fixed when the request starts; no page is reclaimed or added at run time) and
// 落地形态 (compression rules such as H2O run on top unchanged); CAP survey §2.4.1 (3)
// (LM-Infinite / StreamingLLM keep the first tokens and the last L tokens) and (4) (H2O keeps
// the last L tokens plus the tokens with the largest attention accumulated at run time).
//
// Both kernels are small and memory-bound: the append moves 4·D bytes per head; the H2O update
// reads 8 + 4·G bytes and writes 4 per retained token.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <cstdio>

#include "tg.h"
#include "tg_internal.h"

namespace tg {

namespace {

constexpr int kAppendWarps = 8;     // heads per CTA of the append kernel
constexpr int kUpdateThreads = 512;  // threads per head of the H2O update kernel

// Append: one warp per (b, h). Lane 0 picks the slot; the warp copies the K and V rows with
// 16-byte stores (D*2 bytes each); lane 0 updates the head's counters.
//   POLICY 0: sink + recent (head_cursor in/out); POLICY 1: H2O (head_victim in).
template <int POLICY>
__global__ void __launch_bounds__(kAppendWarps * 32)
    append_kernel(int32_t BH, int32_t Hkv, int32_t D, int64_t num_pages, int32_t sink,
                  const uint4 *k_new, const uint4 *v_new, uint4 *k_pages, uint4 *v_pages,
                  const int32_t *table, const int64_t *head_off, const int32_t *budget,
                  int32_t *kv_len, int32_t *cursor, const int32_t *victim, int32_t *slot_pos,
                  float *slot_score, const int32_t *new_pos, int32_t *slot_out) {
    const int32_t bh = blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (bh >= BH) return;
    int32_t slot = -1;
    int64_t pid = -1;
    if (lane == 0) {
        const int32_t bud = budget[bh], n = kv_len[bh];
        if (bud >= 1) {
            if (n < bud) {
                slot = n < 0 ? 0 : n;
            } else if (POLICY == 0) {
                const int32_t s = max(0, min(sink, bud - 1));
                const int32_t R = bud - s;
                int32_t c = cursor[bh] % R;
                if (c < 0) c += R;
                slot = s + c;
            } else {
                const int32_t v = victim[bh];
                slot = (v >= 0 && v < bud) ? v : -1;
            }
        }
        if (slot >= 0) {
            pid = table[head_off[bh] + slot / 16];
            if (pid < 0 || pid >= num_pages) slot = -1;
        }
    }
    slot = __shfl_sync(0xffffffffu, slot, 0);
    pid = __shfl_sync(0xffffffffu, pid, 0);
    if (slot >= 0) {
        const int nvec = D / 8;  // 16-byte vectors per row
        const int64_t dst = (pid * 16 + slot % 16) * nvec;
        const int64_t src = static_cast<int64_t>(bh) * nvec;
        for (int i = lane; i < 2 * nvec; i += 32) {
            if (i < nvec) k_pages[dst + i] = k_new[src + i];
            else v_pages[dst + i - nvec] = v_new[src + i - nvec];
        }
    }
    if (lane == 0) {
        slot_out[bh] = slot;
        if (slot >= 0) {
            const int32_t bud = budget[bh], n = kv_len[bh];
            if (n < bud) {
                kv_len[bh] = slot + 1;
            } else if (POLICY == 0) {
                const int32_t s = max(0, min(sink, bud - 1));
                const int32_t R = bud - s;
                cursor[bh] = (slot - s + 1) % R;
            }
            if (POLICY == 1) {
                const int64_t e = head_off[bh] * 16 + slot;
                slot_pos[e] = new_pos[bh / Hkv];
                slot_score[e] = 0.f;
            }
        }
    }
}

// H2O update: one CTA per (b, h). Adds this step's attention to every retained token's score
// and picks the slot the next token takes: with a free slot, kv_len; else the lowest score among
// tokens older than the last `recent` positions (ties: lowest slot), else the oldest token.
// Each thread takes kUnroll slots per round and issues all their loads before using any, so a
// long head (up to thousands of slots) costs a few dependent rounds, not one per slot.
constexpr int kUnroll = 4;

struct MinPair {
    float s;     // candidate: lowest score ...
    int32_t i;   // ... at the lowest slot
    int32_t p;   // oldest: lowest position ...
    int32_t o;   // ... at the lowest slot
};

__device__ __forceinline__ void take(MinPair &m, float s, int32_t i, int32_t p, int32_t o) {
    if (s < m.s || (s == m.s && i < m.i)) {
        m.s = s;
        m.i = i;
    }
    if (p < m.p || (p == m.p && o < m.o)) {
        m.p = p;
        m.o = o;
    }
}

template <int G4>  // 1: G == 4, token scores read as one 16-byte vector
__global__ void __launch_bounds__(kUpdateThreads)
    h2o_update_kernel(int32_t Hq, int32_t Hkv, int32_t recent, const float *token_scores,
                      const float *lse, const int64_t *head_off, const int32_t *budget,
                      const int32_t *kv_len, const int32_t *slot_pos, float *slot_score,
                      const int32_t *next_pos, int32_t *victim) {
    const int32_t bh = blockIdx.x;
    const int32_t b = bh / Hkv, h = bh - b * Hkv;
    const int32_t G = Hq / Hkv;
    const int32_t n = max(0, kv_len[bh]);
    const int64_t base = head_off[bh] * 16;
    const float *lrow = lse + static_cast<int64_t>(b) * Hq + static_cast<int64_t>(h) * G;
    const int64_t limit = static_cast<int64_t>(next_pos[b]) - recent;
    float l4[4] = {0.f, 0.f, 0.f, 0.f};
    if (G4 && token_scores) {
#pragma unroll
        for (int g = 0; g < 4; ++g) l4[g] = lrow[g];
    }

    MinPair m{INFINITY, 0x7fffffff, 0x7fffffff, 0x7fffffff};
    for (int32_t t0 = threadIdx.x; t0 < n; t0 += kUpdateThreads * kUnroll) {
        float sc[kUnroll];
        int32_t ps[kUnroll];
        float4 tv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int32_t t = t0 + u * kUpdateThreads;
            sc[u] = 0.f;
            ps[u] = 0x7fffffff;
            tv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t < n) {
                sc[u] = slot_score[base + t];
                ps[u] = slot_pos[base + t];
                if (G4 && token_scores) tv[u] = reinterpret_cast<const float4 *>(token_scores)[base + t];
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int32_t t = t0 + u * kUpdateThreads;
            if (t >= n) continue;
            float s = sc[u];
            if (token_scores) {
                if (G4) {
                    s += expf(tv[u].x - l4[0]);
                    s += expf(tv[u].y - l4[1]);
                    s += expf(tv[u].z - l4[2]);
                    s += expf(tv[u].w - l4[3]);
                } else {
                    const float *ts = token_scores + (base + t) * G;
                    for (int32_t g = 0; g < G; ++g) s += expf(ts[g] - lrow[g]);
                }
                slot_score[base + t] = s;
            }
            const bool cand = static_cast<int64_t>(ps[u]) < limit;
            take(m, cand ? s : INFINITY, cand ? t : 0x7fffffff, ps[u], t);
        }
    }
    // (score, slot) and (position, slot) minima: warp shuffles, then one value per warp.
    for (int off = 16; off > 0; off >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, m.s, off);
        const int32_t oi = __shfl_xor_sync(0xffffffffu, m.i, off);
        const int32_t op = __shfl_xor_sync(0xffffffffu, m.p, off);
        const int32_t oo = __shfl_xor_sync(0xffffffffu, m.o, off);
        take(m, os, oi, op, oo);
    }
    __shared__ MinPair wm[kUpdateThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) wm[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kUpdateThreads / 32; ++w) take(m, wm[w].s, wm[w].i, wm[w].p, wm[w].o);
        const int32_t bud = budget[bh];
        int32_t v;
        if (bud < 1) v = -1;
        else if (n < bud) v = n;
        else if (m.i != 0x7fffffff) v = m.i;
        else v = (m.o != 0x7fffffff) ? m.o : -1;
        victim[bh] = v;
    }
}

// Tier migration ("TTKV" 核心方法 1 Tier Layout, 2 Tier Content): one warp per (b, h). The fast
// tier holds the most recent f <= cap tokens, token at position p in fast slot p mod cap; the
// slow tier holds tokens [0, n - f) at slow index = position. A step appends position n: with
// a free fast slot (f < cap, then all tokens are fast: n == f) it takes slot n; with a full
// window the oldest fast token (position n - cap) is quantised (symmetric absmax INT8 per
// token, the rule of tg_quantize_int8) into slow index n - cap, and the new token takes its slot.
// BITS = 8: INT8 codes int8 [row][D]; BITS = 4: INT4 codes packed uint8 [row][D/2], byte i =
// (code_i + 8) | (code_{i+D/2} + 8) << 4 (lane l < 16 packs its values with lane l + 16's).
template <int BITS>
__global__ void __launch_bounds__(kAppendWarps * 32)
    tier_append_kernel(int32_t BH, int32_t D, int64_t num_pages, int64_t num_slow_pages,
                       const __nv_bfloat16 *k_new, const __nv_bfloat16 *v_new,
                       __nv_bfloat16 *k_fast, __nv_bfloat16 *v_fast, const int32_t *fast_table,
                       const int64_t *fast_off, const int32_t *fast_cap, void *k_q8,
                       void *v_q8, float *k_scale, float *v_scale, const int32_t *slow_table,
                       const int64_t *slow_off, const int32_t *slow_cap, int32_t *kv_len,
                       int32_t *fast_len, int32_t *moved_out, int32_t *slot_out) {
    const int32_t bh = blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (bh >= BH) return;
    int32_t fslot = -1, sidx = -1;
    int64_t fpid = -1, spid = -1;
    if (lane == 0) {
        const int32_t n = kv_len[bh], f = fast_len[bh], cap = fast_cap[bh];
        const bool ok = cap >= 1 && f >= 0 && f <= cap && f <= n && (f == cap || n == f);
        if (ok) {
            if (f < cap) {
                fslot = n;
            } else {
                sidx = n - cap;
                fslot = sidx % cap;
                if (sidx >= slow_cap[bh]) fslot = sidx = -1;  // no reserved slow slot left
            }
        }
        if (fslot >= 0) {
            fpid = fast_table[fast_off[bh] + fslot / 16];
            if (fpid < 0 || fpid >= num_pages) fslot = sidx = -1;
        }
        if (sidx >= 0) {
            spid = slow_table[slow_off[bh] + sidx / 16];
            if (spid < 0 || spid >= num_slow_pages) fslot = sidx = -1;
        }
    }
    fslot = __shfl_sync(0xffffffffu, fslot, 0);
    sidx = __shfl_sync(0xffffffffu, sidx, 0);
    fpid = __shfl_sync(0xffffffffu, fpid, 0);
    spid = __shfl_sync(0xffffffffu, spid, 0);
    if (fslot >= 0) {
        const int64_t frow = (fpid * 16 + fslot % 16) * D;
        if (sidx >= 0) {
            // the leaving token's K and V rows -> INT8 / INT4 codes + fp32 scale (read before
            // overwrite)
            const int64_t srow = spid * 16 + sidx % 16;
            constexpr float kLevels = BITS == 4 ? 7.f : 127.f;
            constexpr int kMax = BITS == 4 ? 7 : 127;
            for (int t = 0; t < 2; ++t) {
                const __nv_bfloat16 *src = (t == 0 ? k_fast : v_fast) + frow;
                float x[4];
                float amax = 0.f;
                const int per = D / 32;  // 1..4
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    x[k] = k < per ? __bfloat162float(src[lane * per + k]) : 0.f;
                    amax = fmaxf(amax, fabsf(x[k]));
                }
                for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
                const float sc = __fdiv_rn(amax, kLevels);
                int c[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    c[k] = 0;
                    if (amax != 0.f) c[k] = max(-kMax, min(kMax, __float2int_rn(__fdiv_rn(x[k], sc))));
                }
                if (BITS == 8) {
                    int8_t *codes = static_cast<int8_t *>(t == 0 ? k_q8 : v_q8) + srow * D;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (k < per) codes[lane * per + k] = static_cast<int8_t>(c[k]);
                } else {
                    // d = lane * per + k (< D/2) pairs with d + D/2, held by lane + 16
                    uint8_t *packed = static_cast<uint8_t *>(t == 0 ? k_q8 : v_q8) + srow * (D / 2);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int hi = __shfl_down_sync(0xffffffffu, c[k], 16);
                        if (lane < 16 && k < per)
                            packed[lane * per + k] = static_cast<uint8_t>((c[k] + 8) | ((hi + 8) << 4));
                    }
                }
                if (lane == 0) (t == 0 ? k_scale : v_scale)[srow] = sc;
            }
        }
        __syncwarp();
        const int nvec = D / 8;
        const uint4 *kn = reinterpret_cast<const uint4 *>(k_new) + static_cast<int64_t>(bh) * nvec;
        const uint4 *vn = reinterpret_cast<const uint4 *>(v_new) + static_cast<int64_t>(bh) * nvec;
        uint4 *kd = reinterpret_cast<uint4 *>(k_fast + frow), *vd = reinterpret_cast<uint4 *>(v_fast + frow);
        for (int i = lane; i < 2 * nvec; i += 32) {
            if (i < nvec) kd[i] = kn[i];
            else vd[i - nvec] = vn[i - nvec];
        }
    }
    if (lane == 0) {
        slot_out[bh] = fslot;
        moved_out[bh] = sidx;
        if (fslot >= 0) {
            const int32_t f = fast_len[bh], cap = fast_cap[bh];
            kv_len[bh] = kv_len[bh] + 1;
            fast_len[bh] = f < cap ? f + 1 : cap;
        }
    }
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(const tg_shape *s) {
    if (!s || s->B < 0 || s->Hkv < 1 || s->Hq < s->Hkv || s->Hq % s->Hkv != 0 || s->page != 16 ||
        s->D < 8 || s->D % 8 != 0 || s->num_pages < 0 || static_cast<int64_t>(s->B) * s->Hkv > INT32_MAX)
        return TG_EINVAL;
    return TG_OK;
}

int launch_status(const char *what) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_cuda_error(what, static_cast<int>(e));
        return TG_ECUDA;
    }
    return TG_OK;
}

}  // namespace

}  // namespace tg

using namespace tg;

extern "C" int tg_append_sink_recent(const tg_shape *shape, int32_t sink, const void *k_new,
                                     const void *v_new, void *k_pages, void *v_pages,
                                     const int32_t *page_table, const int64_t *head_page_off,
                                     const int32_t *head_budget, int32_t *head_kv_len,
                                     int32_t *head_cursor, int32_t *slot_out, tg_stream stream) {
    if (check_shape(shape) != TG_OK || sink < 0) return TG_EINVAL;
    const int32_t BH = shape->B * shape->Hkv;
    if (BH == 0) return TG_OK;
    if (!k_new || !v_new || !k_pages || !v_pages || !page_table || !head_page_off ||
        !head_budget || !head_kv_len || !head_cursor || !slot_out || !al16(k_new) ||
        !al16(v_new) || !al16(k_pages) || !al16(v_pages))
        return TG_EINVAL;
    const unsigned grid = static_cast<unsigned>((BH + kAppendWarps - 1) / kAppendWarps);
    append_kernel<0><<<grid, kAppendWarps * 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        BH, shape->Hkv, shape->D, shape->num_pages, sink, static_cast<const uint4 *>(k_new),
        static_cast<const uint4 *>(v_new), static_cast<uint4 *>(k_pages),
        static_cast<uint4 *>(v_pages), page_table, head_page_off, head_budget, head_kv_len,
        head_cursor, nullptr, nullptr, nullptr, nullptr, slot_out);
    return launch_status("append_kernel<sink+recent>");
}

extern "C" int tg_append_h2o(const tg_shape *shape, const void *k_new, const void *v_new,
                             void *k_pages, void *v_pages, const int32_t *page_table,
                             const int64_t *head_page_off, const int32_t *head_budget,
                             int32_t *head_kv_len, const int32_t *head_victim, int32_t *slot_pos,
                             float *slot_score, const int32_t *new_pos, int32_t *slot_out,
                             tg_stream stream) {
    if (check_shape(shape) != TG_OK) return TG_EINVAL;
    const int32_t BH = shape->B * shape->Hkv;
    if (BH == 0) return TG_OK;
    if (!k_new || !v_new || !k_pages || !v_pages || !page_table || !head_page_off ||
        !head_budget || !head_kv_len || !head_victim || !slot_pos || !slot_score || !new_pos ||
        !slot_out || !al16(k_new) || !al16(v_new) || !al16(k_pages) || !al16(v_pages))
        return TG_EINVAL;
    const unsigned grid = static_cast<unsigned>((BH + kAppendWarps - 1) / kAppendWarps);
    append_kernel<1><<<grid, kAppendWarps * 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        BH, shape->Hkv, shape->D, shape->num_pages, 0, static_cast<const uint4 *>(k_new),
        static_cast<const uint4 *>(v_new), static_cast<uint4 *>(k_pages),
        static_cast<uint4 *>(v_pages), page_table, head_page_off, head_budget, head_kv_len,
        nullptr, head_victim, slot_pos, slot_score, new_pos, slot_out);
    return launch_status("append_kernel<h2o>");
}

extern "C" int tg_h2o_update(const tg_shape *shape, int32_t recent, const float *token_scores,
                             const float *lse, const int64_t *head_page_off,
                             const int32_t *head_budget, const int32_t *head_kv_len,
                             const int32_t *slot_pos, float *slot_score, const int32_t *next_pos,
                             int32_t *head_victim, tg_stream stream) {
    if (check_shape(shape) != TG_OK || recent < 0) return TG_EINVAL;
    const int32_t BH = shape->B * shape->Hkv;
    if (BH == 0) return TG_OK;
    if ((token_scores && !lse) || !head_page_off || !head_budget || !head_kv_len || !slot_pos ||
        !slot_score || !next_pos || !head_victim)
        return TG_EINVAL;
    const bool g4 = shape->Hq / shape->Hkv == 4 &&
                    (reinterpret_cast<uintptr_t>(token_scores) & 15u) == 0;
    auto kern = g4 ? h2o_update_kernel<1> : h2o_update_kernel<0>;
    kern<<<static_cast<unsigned>(BH), kUpdateThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        shape->Hq, shape->Hkv, recent, token_scores, lse, head_page_off, head_budget, head_kv_len,
        slot_pos, slot_score, next_pos, head_victim);
    return launch_status("h2o_update_kernel");
}

namespace tg {
namespace {

template <int BITS>
int tiered_append(const tg_shape *shape, const void *k_new, const void *v_new, void *k_fast, void *v_fast,
                  const int32_t *fast_page_table, const int64_t *fast_head_off, const int32_t *head_fast_cap,
                  void *k_codes, void *v_codes, float *k_scale, float *v_scale, const int32_t *slow_page_table,
                  const int64_t *slow_head_off, const int32_t *head_slow_cap, int32_t *head_kv_len,
                  int32_t *head_fast_len, int32_t *moved_out, int32_t *slot_out, tg_stream stream) {
    if (check_shape(shape) != TG_OK || shape->D % 32 != 0 || shape->D > 128 ||
        shape->num_slow_pages < 0)
        return TG_EINVAL;
    const int32_t BH = shape->B * shape->Hkv;
    if (BH == 0) return TG_OK;
    if (!k_new || !v_new || !k_fast || !v_fast || !fast_page_table || !fast_head_off ||
        !head_fast_cap || !k_codes || !v_codes || !k_scale || !v_scale || !slow_page_table ||
        !slow_head_off || !head_slow_cap || !head_kv_len || !head_fast_len || !moved_out ||
        !slot_out || !al16(k_new) || !al16(v_new) || !al16(k_fast) || !al16(v_fast))
        return TG_EINVAL;
    const unsigned grid = static_cast<unsigned>((BH + kAppendWarps - 1) / kAppendWarps);
    tier_append_kernel<BITS><<<grid, kAppendWarps * 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        BH, shape->D, shape->num_pages, shape->num_slow_pages,
        static_cast<const __nv_bfloat16 *>(k_new), static_cast<const __nv_bfloat16 *>(v_new),
        static_cast<__nv_bfloat16 *>(k_fast), static_cast<__nv_bfloat16 *>(v_fast), fast_page_table,
        fast_head_off, head_fast_cap, k_codes, v_codes, k_scale, v_scale, slow_page_table, slow_head_off,
        head_slow_cap, head_kv_len, head_fast_len, moved_out, slot_out);
    return launch_status("tier_append_kernel");
}

}  // namespace
}  // namespace tg

extern "C" int tg_tiered_append(const tg_shape *shape, const void *k_new, const void *v_new,
                                void *k_fast, void *v_fast, const int32_t *fast_page_table,
                                const int64_t *fast_head_off, const int32_t *head_fast_cap,
                                int8_t *k_q8, int8_t *v_q8, float *k_scale, float *v_scale,
                                const int32_t *slow_page_table, const int64_t *slow_head_off,
                                const int32_t *head_slow_cap, int32_t *head_kv_len,
                                int32_t *head_fast_len, int32_t *moved_out, int32_t *slot_out,
                                tg_stream stream) {
    return tg::tiered_append<8>(shape, k_new, v_new, k_fast, v_fast, fast_page_table, fast_head_off,
                                head_fast_cap, k_q8, v_q8, k_scale, v_scale, slow_page_table, slow_head_off,
                                head_slow_cap, head_kv_len, head_fast_len, moved_out, slot_out, stream);
}

extern "C" int tg_tiered_append_int4(const tg_shape *shape, const void *k_new, const void *v_new,
                                     void *k_fast, void *v_fast, const int32_t *fast_page_table,
                                     const int64_t *fast_head_off, const int32_t *head_fast_cap,
                                     uint8_t *k_q4, uint8_t *v_q4, float *k_scale, float *v_scale,
                                     const int32_t *slow_page_table, const int64_t *slow_head_off,
                                     const int32_t *head_slow_cap, int32_t *head_kv_len,
                                     int32_t *head_fast_len, int32_t *moved_out, int32_t *slot_out,
                                     tg_stream stream) {
    return tg::tiered_append<4>(shape, k_new, v_new, k_fast, v_fast, fast_page_table, fast_head_off,
                                head_fast_cap, k_q4, v_q4, k_scale, v_scale, slow_page_table, slow_head_off,
                                head_slow_cap, head_kv_len, head_fast_len, moved_out, slot_out, stream);
}
