// SplitZip: lossless BF16 codec for KV transfer ("SplitZip" explainer, arXiv 2605.01708,
// "Die SplitZip-Strategie" and "Warum es schnell ist"). A bf16 value is sign, 8-bit exponent
// and 7-bit mantissa; the 16 most frequent exponents get 4-bit codes packed two per byte, rare
// exponents go to an escape stream (position, exponent) that decoding applies as overwrites.
// Layout: codebook uint8[16] (count descending, ties by exponent ascending, over all 256
// exponents); sm uint8[n] = (sign << 7) | mantissa; codes uint8[(n+1)/2], element i in byte i/2,
// low nibble for even i; escaped elements carry code 0; escapes in ascending position.
//
// Every kernel is HBM-bound and grid-sized in tiles: encode reads 2 B per element twice
// (histogram, encode) and writes 1.5 B; decode reads 1.5 B and writes 2 B. The encode pass
// leaves, for tiles that hold escapes, one 16-bit escape mask per thread, and per-group escape
// totals; one escape pass then places every tile's escapes from those alone (no second read of
// the source beyond the escaped elements, no separate scan kernel).
#include <cuda_runtime.h>
#include <stdint.h>

#include "tg.h"
#include "tg_internal.h"

namespace tg {
namespace {

constexpr int kZipThreads = 256;
constexpr int kZipPer = 16;                        // elements per thread
constexpr int kZipTile = kZipThreads * kZipPer;    // elements per tile (one CTA)
constexpr int kZipHistBlocks = 4 * 148;
constexpr int kZipGroups = 8 * 148;               // escape-pass CTAs, one per group of tiles

// Workspace: histogram u64[256] | group escape totals u64[kZipGroups] (both zeroed by one
// memset) | exponent -> code u8[256] | per-tile escape counts u32[T] | per-thread escape masks
// u16[T * kZipThreads] (T tiles; masks are written only for tiles that hold escapes).
constexpr int64_t kZipZeroBytes = 2048 + 8 * kZipGroups;
constexpr int64_t kZipLutAt = kZipZeroBytes;
constexpr int64_t kZipCountAt = kZipLutAt + 256;

struct ZipWs {
    unsigned long long *hist;
    unsigned long long *group_sum;
    uint8_t *lut;
    uint32_t *tile_count;
    uint16_t *masks;
};

int64_t zip_tiles(int64_t n) { return (n + kZipTile - 1) / kZipTile; }
int64_t pad256(int64_t b) { return (b + 255) / 256 * 256; }

ZipWs zip_ws(void *ws, int64_t n) {
    char *p = static_cast<char *>(ws);
    const int64_t T = zip_tiles(n);
    ZipWs w;
    w.hist = reinterpret_cast<unsigned long long *>(p);
    w.group_sum = reinterpret_cast<unsigned long long *>(p + 2048);
    w.lut = reinterpret_cast<uint8_t *>(p + kZipLutAt);
    w.tile_count = reinterpret_cast<uint32_t *>(p + kZipCountAt);
    w.masks = reinterpret_cast<uint16_t *>(p + kZipCountAt + pad256(T * 4));
    return w;
}

__device__ __forceinline__ uint32_t zexp(uint32_t x) { return (x >> 7) & 0xFFu; }

constexpr uint8_t kZipEsc = 0x10;  // lut entry of an escaped exponent: code 0, bit 4 set

__global__ void __launch_bounds__(kZipThreads) zip_hist_kernel(int64_t n, const uint16_t *src,
                                                                unsigned long long *hist) {
    __shared__ uint32_t h[256];
    h[threadIdx.x] = 0;
    __syncthreads();
    const int64_t nv = n / 8;
    const uint4 *v = reinterpret_cast<const uint4 *>(src);
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kZipThreads + threadIdx.x; i < nv;
         i += static_cast<int64_t>(gridDim.x) * kZipThreads) {
        const uint4 w = v[i];
        const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            atomicAdd(&h[zexp(words[k])], 1u);
            atomicAdd(&h[zexp(words[k] >> 16)], 1u);
        }
    }
    if (blockIdx.x == 0)
        for (int64_t i = nv * 8 + threadIdx.x; i < n; i += kZipThreads) atomicAdd(&h[zexp(src[i])], 1u);
    __syncthreads();
    if (h[threadIdx.x]) atomicAdd(&hist[threadIdx.x], static_cast<unsigned long long>(h[threadIdx.x]));
}

// One block: exponent e's rank = exponents with a larger count, or the same count and a
// smaller value; ranks 0..15 are the codebook. lut[e] = its code, or kZipEsc (code bits 0) for
// an exponent outside the codebook.
__global__ void __launch_bounds__(256) zip_codebook_kernel(const unsigned long long *hist,
                                                           uint8_t *codebook, uint8_t *lut) {
    __shared__ unsigned long long c[256];
    const int e = threadIdx.x;
    c[e] = hist[e];
    __syncthreads();
    int rank = 0;
    for (int f = 0; f < 256; ++f) rank += (c[f] > c[e] || (c[f] == c[e] && f < e)) ? 1 : 0;
    if (rank < 16) codebook[rank] = static_cast<uint8_t>(e);
    lut[e] = rank < 16 ? static_cast<uint8_t>(rank) : kZipEsc;
}

// Tile `blockIdx.x` belongs to group blockIdx.x / tpg.
__global__ void __launch_bounds__(kZipThreads) zip_encode_kernel(int64_t n, int64_t tpg, const uint16_t *src,
                                                                  const uint8_t *lut_g, uint8_t *sm,
                                                                  uint8_t *codes, uint32_t *tile_count,
                                                                  uint16_t *masks,
                                                                  unsigned long long *group_sum) {
    __shared__ uint8_t lut[256];
    __shared__ uint32_t wsum[kZipThreads / 32];
    lut[threadIdx.x] = lut_g[threadIdx.x];
    __syncthreads();
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * kZipTile + static_cast<int64_t>(threadIdx.x) * kZipPer;
    uint32_t flags = 0;  // bit k: element i0 + k escapes
    if (i0 + kZipPer <= n) {
        const uint4 a = reinterpret_cast<const uint4 *>(src + i0)[0];
        const uint4 b = reinterpret_cast<const uint4 *>(src + i0)[1];
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        // Four elements per step on packed bytes: hi = sign | exponent bits 7..1, lo = exponent
        // bit 0 | mantissa, byte i of each for element 4j + i.
        uint32_t s[4], ex[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t hi = __byte_perm(w[2 * j], w[2 * j + 1], 0x7531);
            const uint32_t lo = __byte_perm(w[2 * j], w[2 * j + 1], 0x6420);
            s[j] = (hi & 0x80808080u) | (lo & 0x7F7F7F7Fu);
            ex[j] = ((hi << 1) & 0xFEFEFEFEu) | ((lo >> 7) & 0x01010101u);
        }
        // lut values (< 32) of even elements 2m go to byte m of ve, odd ones to byte m of vo;
        // a code word is then the low nibbles of both, interleaved.
        uint32_t ve[2] = {0u, 0u}, vo[2] = {0u, 0u};
#pragma unroll
        for (int k = 0; k < kZipPer; ++k) {
            const uint32_t e = __byte_perm(ex[k >> 2], 0u, 0x4440 + (k & 3));
            const uint32_t v = lut[e];
            const uint32_t at = 1u << (8 * ((k >> 1) & 3));
            if (k & 1)
                vo[k >> 3] += v * at;
            else
                ve[k >> 3] += v * at;
        }
        uint32_t c[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) c[h] = (ve[h] & 0x0F0F0F0Fu) | ((vo[h] << 4) & 0xF0F0F0F0u);
        if (((ve[0] | ve[1] | vo[0] | vo[1]) & 0x10101010u) != 0u) {
#pragma unroll
            for (int k = 0; k < kZipPer; ++k)
                flags |= ((static_cast<uint32_t>(lut[__byte_perm(ex[k >> 2], 0u, 0x4440 + (k & 3))]) >> 4) & 1u) << k;
        }
        reinterpret_cast<uint4 *>(sm + i0)[0] = make_uint4(s[0], s[1], s[2], s[3]);
        reinterpret_cast<uint2 *>(codes + i0 / 2)[0] = make_uint2(c[0], c[1]);
    } else if (i0 < n) {
        for (int64_t i = i0; i < n; i += 2) {
            uint32_t byte = 0;
            for (int k = 0; k < 2 && i + k < n; ++k) {
                const uint32_t x = src[i + k];
                sm[i + k] = static_cast<uint8_t>(((x >> 15) << 7) | (x & 0x7Fu));
                const uint32_t v = lut[zexp(x)];
                if (v & kZipEsc) flags |= 1u << (i + k - i0);
                byte |= (v & 0xFu) << (4 * k);
            }
            codes[i / 2] = static_cast<uint8_t>(byte);
        }
    }
    uint32_t esc = __popc(flags);
    for (int off = 16; off > 0; off >>= 1) esc += __shfl_xor_sync(0xffffffffu, esc, off);
    if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = esc;
    __syncthreads();
    uint32_t t = 0;
    for (int w = 0; w < kZipThreads / 32; ++w) t += wsum[w];
    if (t) masks[static_cast<int64_t>(blockIdx.x) * kZipThreads + threadIdx.x] = static_cast<uint16_t>(flags);
    if (threadIdx.x == 0) {
        tile_count[blockIdx.x] = t;
        if (t) atomicAdd(&group_sum[blockIdx.x / tpg], static_cast<unsigned long long>(t));
    }
}

// One warp places the escapes of one tile, in ascending position, from `at`. Lane l reads the
// masks of threads 8l..8l+7, which cover the tile's elements 128l..128l+127 in order.
__device__ void zip_escape_tile(int64_t tile, int64_t at, const uint16_t *src, const uint16_t *masks,
                                int64_t *esc_pos, uint8_t *esc_exp, int64_t esc_cap) {
    const int lane = threadIdx.x & 31;
    const uint4 m = reinterpret_cast<const uint4 *>(masks + tile * kZipThreads)[lane];
    const uint32_t mw[4] = {m.x, m.y, m.z, m.w};
    const uint32_t mine = __popc(m.x) + __popc(m.y) + __popc(m.z) + __popc(m.w);
    uint32_t incl = mine;
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    at += incl - mine;
    const int64_t e0 = tile * kZipTile + static_cast<int64_t>(lane) * 8 * kZipPer;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        // word q: masks of threads 8l+2q (low half) and 8l+2q+1 (high half) = elements 32q+b
        for (uint32_t bits = mw[q]; bits; bits &= bits - 1) {
            const int64_t i = e0 + 32 * q + (__ffs(bits) - 1);
            if (at < esc_cap) {
                esc_pos[at] = i;
                esc_exp[at] = static_cast<uint8_t>(zexp(src[i]));
            }
            ++at;
        }
    }
}

// Block g owns tiles [g*tpg, (g+1)*tpg): its base offset is the sum of the earlier groups'
// totals; chunks of 256 tile counts are scanned in shared memory and each warp places the
// escapes of the chunk's tiles that hold any. Block 0 writes the total escape count.
__global__ void __launch_bounds__(kZipThreads) zip_escape_kernel(int64_t T, int64_t tpg, int ng,
                                                                  const uint16_t *src,
                                                                  const unsigned long long *group_sum,
                                                                  const uint32_t *tile_count,
                                                                  const uint16_t *masks, int64_t *esc_pos,
                                                                  uint8_t *esc_exp, int64_t esc_cap,
                                                                  int64_t *n_esc) {
    __shared__ unsigned long long red[2][kZipThreads / 32];
    __shared__ int64_t toff[kZipThreads];
    __shared__ uint32_t tcnt[kZipThreads];
    __shared__ uint32_t wsum[kZipThreads / 32];
    const int g = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned long long before = 0, total = 0;
    for (int h = threadIdx.x; h < ng; h += kZipThreads) {
        const unsigned long long v = group_sum[h];
        total += v;
        if (h < g) before += v;
    }
    for (int off = 16; off > 0; off >>= 1) {
        before += __shfl_xor_sync(0xffffffffu, before, off);
        total += __shfl_xor_sync(0xffffffffu, total, off);
    }
    if (lane == 0) {
        red[0][warp] = before;
        red[1][warp] = total;
    }
    __syncthreads();
    int64_t carry = 0, all = 0;
    for (int w = 0; w < kZipThreads / 32; ++w) {
        carry += static_cast<int64_t>(red[0][w]);
        all += static_cast<int64_t>(red[1][w]);
    }
    if (g == 0 && threadIdx.x == 0) *n_esc = all;
    const int64_t t0 = static_cast<int64_t>(g) * tpg;
    const int64_t t1 = t0 + tpg < T ? t0 + tpg : T;
    for (int64_t c0 = t0; c0 < t1; c0 += kZipThreads) {
        const int64_t t = c0 + threadIdx.x;
        const uint32_t cnt = t < t1 ? tile_count[t] : 0u;
        uint32_t incl = cnt;
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        uint32_t wbefore = 0, chunk = 0;
        for (int w = 0; w < kZipThreads / 32; ++w) {
            wbefore += w < warp ? wsum[w] : 0u;
            chunk += wsum[w];
        }
        toff[threadIdx.x] = carry + wbefore + incl - cnt;
        tcnt[threadIdx.x] = cnt;
        __syncthreads();
        const int64_t nt = t1 - c0 < kZipThreads ? t1 - c0 : kZipThreads;
        for (int j = warp; j < nt; j += kZipThreads / 32)
            if (tcnt[j]) zip_escape_tile(c0 + j, toff[j], src, masks, esc_pos, esc_exp, esc_cap);
        carry += chunk;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kZipThreads) zip_decode_kernel(int64_t n, const uint8_t *codebook_g,
                                                                  const uint8_t *sm, const uint8_t *codes,
                                                                  uint16_t *dst) {
    __shared__ uint32_t cb[16];
    if (threadIdx.x < 16) cb[threadIdx.x] = codebook_g[threadIdx.x];
    __syncthreads();
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * kZipTile + static_cast<int64_t>(threadIdx.x) * kZipPer;
    if (i0 + kZipPer <= n) {
        const uint4 s = reinterpret_cast<const uint4 *>(sm + i0)[0];
        const uint2 c = reinterpret_cast<const uint2 *>(codes + i0 / 2)[0];
        const uint32_t sw[4] = {s.x, s.y, s.z, s.w}, cw[2] = {c.x, c.y};
        uint32_t o[8];
#pragma unroll
        for (int k = 0; k < kZipPer; k += 2) {
            uint32_t pair = 0;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint32_t b = (sw[(k + u) >> 2] >> (8 * ((k + u) & 3))) & 0xFFu;
                const uint32_t e = cb[(cw[(k + u) >> 3] >> (4 * ((k + u) & 7))) & 0xFu];
                pair |= (((b >> 7) << 15) | (e << 7) | (b & 0x7Fu)) << (16 * u);
            }
            o[k >> 1] = pair;
        }
        reinterpret_cast<uint4 *>(dst + i0)[0] = make_uint4(o[0], o[1], o[2], o[3]);
        reinterpret_cast<uint4 *>(dst + i0)[1] = make_uint4(o[4], o[5], o[6], o[7]);
    } else {
        for (int64_t i = i0; i < n; ++i) {
            const uint32_t b = sm[i];
            const uint32_t e = cb[(codes[i / 2] >> (4 * (i & 1))) & 0xFu];
            dst[i] = static_cast<uint16_t>(((b >> 7) << 15) | (e << 7) | (b & 0x7Fu));
        }
    }
}

__global__ void zip_apply_escapes_kernel(const int64_t *n_esc, int64_t esc_cap, const int64_t *esc_pos,
                                         const uint8_t *esc_exp, int64_t n, uint16_t *dst) {
    const int64_t k = *n_esc < esc_cap ? *n_esc : esc_cap;
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < k;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = esc_pos[j];
        if (i >= 0 && i < n) dst[i] = static_cast<uint16_t>((dst[i] & 0x807Fu) | (static_cast<uint32_t>(esc_exp[j]) << 7));
    }
}

bool al(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int zip_launch_status(const char *what) {
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

extern "C" int64_t tg_splitzip_workspace_bytes(int64_t n) {
    if (n < 0) return -1;
    const int64_t T = zip_tiles(n);
    return kZipCountAt + pad256(T * 4) + pad256(T * kZipThreads * 2);
}

extern "C" int tg_splitzip_encode(int64_t n, const void *src, uint8_t *codebook, uint8_t *sm,
                                  uint8_t *codes, int64_t *esc_pos, uint8_t *esc_exp,
                                  int64_t esc_cap, int64_t *n_esc, void *workspace,
                                  tg_stream stream_) {
    if (n < 0 || esc_cap < 0 || !codebook || !n_esc || !workspace) return TG_EINVAL;
    if (n > 0 && (!src || !sm || !codes || !al(src, 16) || !al(sm, 16) || !al(codes, 8) ||
                  !al(workspace, 256) || (esc_cap > 0 && (!esc_pos || !esc_exp))))
        return TG_EINVAL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    const ZipWs w = zip_ws(workspace, n);
    const int64_t T = zip_tiles(n);
    if (cudaMemsetAsync(w.hist, 0, kZipZeroBytes, stream) != cudaSuccess) return zip_launch_status("cudaMemsetAsync");
    const uint16_t *x = static_cast<const uint16_t *>(src);
    const int64_t hb = n / 8 / kZipThreads + 1;
    zip_hist_kernel<<<static_cast<unsigned>(hb < kZipHistBlocks ? hb : kZipHistBlocks), kZipThreads, 0, stream>>>(n, x, w.hist);
    zip_codebook_kernel<<<1, 256, 0, stream>>>(w.hist, codebook, w.lut);
    if (T > 0) {
        const int64_t tpg = (T + kZipGroups - 1) / kZipGroups;
        const int ng = static_cast<int>((T + tpg - 1) / tpg);
        zip_encode_kernel<<<static_cast<unsigned>(T), kZipThreads, 0, stream>>>(n, tpg, x, w.lut, sm, codes,
                                                                            w.tile_count, w.masks, w.group_sum);
        zip_escape_kernel<<<static_cast<unsigned>(ng), kZipThreads, 0, stream>>>(
            T, tpg, ng, x, w.group_sum, w.tile_count, w.masks, esc_pos, esc_exp, esc_cap, n_esc);
    } else if (cudaMemsetAsync(n_esc, 0, sizeof(int64_t), stream) != cudaSuccess) {
        return zip_launch_status("cudaMemsetAsync");
    }
    return zip_launch_status("splitzip encode kernels");
}

extern "C" int tg_splitzip_decode(int64_t n, const uint8_t *codebook, const uint8_t *sm,
                                  const uint8_t *codes, const int64_t *esc_pos,
                                  const uint8_t *esc_exp, const int64_t *n_esc, int64_t esc_cap,
                                  void *dst, tg_stream stream_) {
    if (n < 0 || esc_cap < 0 || !codebook || !n_esc) return TG_EINVAL;
    if (n == 0) return TG_OK;
    if (!sm || !codes || !dst || !al(dst, 16) || !al(sm, 16) || !al(codes, 8) ||
        (esc_cap > 0 && (!esc_pos || !esc_exp)))
        return TG_EINVAL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    uint16_t *y = static_cast<uint16_t *>(dst);
    zip_decode_kernel<<<static_cast<unsigned>(zip_tiles(n)), kZipThreads, 0, stream>>>(n, codebook, sm, codes, y);
    if (esc_cap > 0) zip_apply_escapes_kernel<<<148, 256, 0, stream>>>(n_esc, esc_cap, esc_pos, esc_exp, n, y);
    return zip_launch_status("splitzip decode kernels");
}
