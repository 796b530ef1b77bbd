"""Seeded synthetic inputs for the paged decode workloads.

Holds random draws and workload shapes only: no retained-length rule, no budget grouping, no
page allocation, no quantisation and no attention arithmetic. Those belong to the method and
are implemented twice, independently: once in the CUDA library and once in the CPU oracle.
Both receive the bytes produced here.

Every value is a pure function of (seed, stream, index) through counter-based SplitMix64
(Steele, Lea & Flood, OOPSLA 2014); see synth.c. Streams are named by ``stream_id``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, replace
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "_libsynth.so")
_lib = None

# Stream kinds. A stream id is (kind << 32) | sub, sub = layer (or 0).
S_LEN = 1        # full context length L_b per sequence, or direct retained length per head
S_RANK = 2       # head-importance ranking permutation (the synthetic budget table)
S_JITTER = 3     # per-(sequence, head) ratio jitter
S_FREE = 4       # initial free-list order of the page pool
S_DOC = 5        # prefix layout: which shared document a sequence extends
S_SUFFIX = 6     # prefix layout: private suffix length
S_Q = 7          # query rows
S_K = 8          # K page contents (bf16 pool)
S_V = 9          # V page contents (bf16 pool)
S_KSLOW = 10     # K contents of slow-tier pages before INT8 quantisation
S_VSLOW = 11     # V contents of slow-tier pages before INT8 quantisation
S_FREE_SLOW = 12 # free-list order of the slow-tier pool
S_NEWK = 13      # K row of the token a decode step appends (sub = step)
S_NEWV = 14      # V row of the token a decode step appends (sub = step)
S_SCORE = 15     # initial accumulated attention score of each retained slot (H2O)
S_PICK = 16      # which older positions a head retained at admission (H2O)


def stream_id(kind: int, sub: int = 0) -> int:
    return (int(kind) << 32) | int(sub)


def build(force: bool = False) -> str:
    """Compile synth.c into _libsynth.so (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC,
                               "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        u64, i64, p = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        lib.synth_stream_key.restype = u64
        lib.synth_stream_key.argtypes = [u64, u64]
        lib.synth_draw.restype = u64
        lib.synth_draw.argtypes = [u64, u64, u64]
        lib.synth_draws.argtypes = [u64, u64, u64, i64, p]
        lib.synth_uniform_int.argtypes = [u64, u64, u64, i64, i64, i64, p]
        lib.synth_normal_bf16.argtypes = [u64, u64, u64, i64, ctypes.c_double, ctypes.c_double, p]
        lib.synth_normal_f64.argtypes = [u64, u64, u64, i64, p]
        lib.synth_permutation.argtypes = [u64, u64, i64, p]
        _lib = lib
    return _lib


def stream_key(seed: int, stream: int) -> int:
    """The SplitMix64 seed of a stream: its draw i is the (i+1)-th output of SplitMix64 seeded
    with this value (so a consumer holding its own SplitMix64 can replay the stream)."""
    return int(_L().synth_stream_key(seed, stream))


def draws(seed: int, stream: int, n: int, i0: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _L().synth_draws(seed, stream, i0, n, out.ctypes.data)
    return out


def uniform_int(seed: int, stream: int, n: int, lo: int, hi: int, i0: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _L().synth_uniform_int(seed, stream, i0, n, lo, hi, out.ctypes.data)
    return out


def normal_bf16(seed: int, stream: int, n: int, i0: int = 0, mean: float = 0.0,
                sd: float = 1.0, out: Optional[np.ndarray] = None) -> np.ndarray:
    """n bf16 normals as raw uint16 bits (view as torch.bfloat16 / widen with bf16_to_f64)."""
    if out is None:
        out = np.empty(n, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.size == n and out.flags.c_contiguous
    _L().synth_normal_bf16(seed, stream, i0, n, mean, sd, out.ctypes.data)
    return out


def normal_f64(seed: int, stream: int, n: int, i0: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _L().synth_normal_f64(seed, stream, i0, n, out.ctypes.data)
    return out


def permutation(seed: int, stream: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _L().synth_permutation(seed, stream, n, out.ctypes.data)
    return out


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round to float32 then to bf16 (RNE) bits; for building small hand-made inputs."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


# ----------------------------------------------------------------------------------------
# Workload specs (shapes and distributions of the five decode workloads).
# ----------------------------------------------------------------------------------------

@dataclass(frozen=True)
class Spec:
    """Shape and distribution of one synthetic decode workload.

    kind:
      "direct"  retained length per (sequence, KV head) drawn uniformly in [len_lo, len_hi]
      "ratio"   full context L_b uniform in [len_lo, len_hi]; retention ratio (ppm) per
                (sequence, KV head) = budget-table entry of the head + uniform jitter,
                clamped to [ratio_lo_ppm, ratio_hi_ppm]
      "prefix"  shared system segment + one of n_docs shared document segments + private
                suffix uniform in [suffix_lo, suffix_hi]; full retention
      "tiered"  full retention of len_lo tokens; the last fast_tokens in bf16, the rest
                quantised to INT8
    """
    name: str
    kind: str
    B: int
    Hq: int
    Hkv: int
    D: int
    layers: int = 1
    page: int = 16
    len_lo: int = 0
    len_hi: int = 0
    ratio_lo_ppm: int = 0
    ratio_hi_ppm: int = 0
    jitter_ppm: int = 0
    rank_over_layers: bool = False
    groups: int = 1
    occupancy_num: int = 1      # num_pages = floor(used * num / den)
    occupancy_den: int = 1
    sys_tokens: int = 0
    n_docs: int = 0
    doc_tokens: int = 0
    suffix_lo: int = 0
    suffix_hi: int = 0
    fast_tokens: int = 0
    seed: int = 0x7A4E0000
    slow_bits: int = 8          # tiered: code width of the slow tier (8 or 4)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))


def preset(cfg: int) -> Spec:
    """The five decode workloads at full size (cfg = 1..5)."""
    s = 0x7A4E0000 + cfg
    if cfg == 1:
        return Spec("tiny ragged MHA decode", "direct", B=1, Hq=8, Hkv=8, D=64,
                    len_lo=16, len_hi=256, groups=1, seed=s)
    if cfg == 2:
        return Spec("GQA decode layer, ragged budgets", "ratio", B=64, Hq=32, Hkv=8, D=128,
                    len_lo=2048, len_hi=8192, ratio_lo_ppm=100_000, ratio_hi_ppm=900_000,
                    jitter_ppm=50_000, groups=4, occupancy_num=10, occupancy_den=9, seed=s)
    if cfg == 3:
        return Spec("multi-turn serving step", "ratio", B=256, Hq=32, Hkv=8, D=128, layers=32,
                    len_lo=4096, len_hi=32768, ratio_lo_ppm=50_000, ratio_hi_ppm=500_000,
                    jitter_ppm=0, rank_over_layers=True, groups=8, occupancy_num=10,
                    occupancy_den=9, seed=s)
    if cfg == 4:
        return Spec("prefix-shared decode", "prefix", B=512, Hq=32, Hkv=8, D=128,
                    sys_tokens=2000, n_docs=8, doc_tokens=500, suffix_lo=80, suffix_hi=100,
                    groups=1, seed=s)
    if cfg == 5:
        return Spec("tiered long-context decode", "tiered", B=4, Hq=32, Hkv=8, D=128,
                    len_lo=131072, len_hi=131072, fast_tokens=8192, groups=1, seed=s)
    raise ValueError(cfg)


def small(cfg: int, **over) -> Spec:
    """Reduced variants of the presets that the oracle finishes in seconds, still spanning
    several pages per head, several splits and a ragged tail page."""
    base = preset(cfg)
    if cfg == 1:
        sp = base
    elif cfg == 2:
        sp = replace(base, B=6, len_lo=300, len_hi=1500)
    elif cfg == 3:
        sp = replace(base, B=5, layers=3, Hq=16, Hkv=4, len_lo=400, len_hi=3000, groups=4)
    elif cfg == 4:
        sp = replace(base, B=12, sys_tokens=200, n_docs=3, doc_tokens=50, suffix_lo=8,
                     suffix_hi=40)
    elif cfg == 5:
        sp = replace(base, B=2, len_lo=2100, len_hi=2100, fast_tokens=300)
    else:
        raise ValueError(cfg)
    return replace(sp, **over) if over else sp


# ----------------------------------------------------------------------------------------
# Draws that define a workload instance (all "given" quantities; the method's arithmetic is
# applied by whoever consumes them).
# ----------------------------------------------------------------------------------------

def full_lengths(sp: Spec, layer: int = 0) -> np.ndarray:
    """"ratio"/"tiered": full context length L_b per sequence, int32[B] (same for all layers)."""
    if sp.kind == "tiered":
        return np.full(sp.B, sp.len_lo, dtype=np.int32)
    return uniform_int(sp.seed, stream_id(S_LEN), sp.B, sp.len_lo, sp.len_hi)


def direct_lengths(sp: Spec, layer: int = 0) -> np.ndarray:
    """"direct": retained length per (sequence, KV head), int32[B, Hkv]."""
    return uniform_int(sp.seed, stream_id(S_LEN, layer), sp.B * sp.Hkv, sp.len_lo,
                       sp.len_hi).reshape(sp.B, sp.Hkv)


def budget_table_ppm(sp: Spec) -> np.ndarray:
    """Synthetic stand-in for the offline-calibrated budget table: a seeded head-importance
    ranking mapped linearly onto [ratio_lo_ppm, ratio_hi_ppm]. int32[layers, Hkv].

    With rank_over_layers the ranking runs over all (layer, KV head) pairs, otherwise over
    the KV heads of one layer (the same table for every layer)."""
    R = sp.layers * sp.Hkv if sp.rank_over_layers else sp.Hkv
    rank = permutation(sp.seed, stream_id(S_RANK), R).astype(np.int64)
    lo, hi = sp.ratio_lo_ppm, sp.ratio_hi_ppm
    if R == 1:
        ppm = np.full(1, lo, dtype=np.int64)
    else:
        ppm = lo + ((hi - lo) * rank + (R - 1) // 2) // (R - 1)
    if sp.rank_over_layers:
        return ppm.reshape(sp.layers, sp.Hkv).astype(np.int32)
    return np.tile(ppm.reshape(1, sp.Hkv), (sp.layers, 1)).astype(np.int32)


def ratio_ppm(sp: Spec, layer: int = 0) -> np.ndarray:
    """Per-(sequence, KV head) retention ratio in ppm: budget-table entry + jitter, clamped.
    int32[B, Hkv]."""
    base = budget_table_ppm(sp)[layer].astype(np.int64)
    r = np.tile(base.reshape(1, sp.Hkv), (sp.B, 1))
    if sp.jitter_ppm:
        j = uniform_int(sp.seed, stream_id(S_JITTER, layer), sp.B * sp.Hkv, -sp.jitter_ppm,
                        sp.jitter_ppm).reshape(sp.B, sp.Hkv)
        r = np.clip(r + j, sp.ratio_lo_ppm, sp.ratio_hi_ppm)
    return r.astype(np.int32)


def prefix_layout(sp: Spec):
    """"prefix": (doc index per sequence int32[B], private suffix length int32[B])."""
    doc = (draws(sp.seed, stream_id(S_DOC), sp.B) % np.uint64(sp.n_docs)).astype(np.int32)
    suf = uniform_int(sp.seed, stream_id(S_SUFFIX), sp.B, sp.suffix_lo, sp.suffix_hi)
    return doc, suf


def free_order(sp: Spec, num_pages: int, layer: int = 0, slow: bool = False) -> np.ndarray:
    """Initial free-list order of a pool of num_pages pages (a seeded shuffle)."""
    return permutation(sp.seed, stream_id(S_FREE_SLOW if slow else S_FREE, layer), num_pages)


def free_order_seed(sp: Spec, layer: int = 0, slow: bool = False) -> int:
    """SplitMix64 seed of the free-order stream: an allocator that shuffles its pool itself
    (Fisher-Yates driven by SplitMix64 from this seed) reproduces free_order."""
    return stream_key(sp.seed, stream_id(S_FREE_SLOW if slow else S_FREE, layer))


def q_bits(sp: Spec, layer: int = 0) -> np.ndarray:
    """Query rows, bf16 bits uint16[B, Hq, D], N(0, 1)."""
    n = sp.B * sp.Hq * sp.D
    return normal_bf16(sp.seed, stream_id(S_Q, layer), n).reshape(sp.B, sp.Hq, sp.D)


def pool_bits(sp: Spec, which: str, num_pages: int,
              out: Optional[np.ndarray] = None) -> np.ndarray:
    """Page-pool contents as bf16 bits uint16[num_pages, page, D], N(0, 1) per element,
    a pure function of (physical page, slot, dim). which in {"k", "v", "kslow", "vslow"}.
    The contents do not depend on the layer: every layer's pool holds the same bytes, and
    the layer's own tables decide which pages (and so which values) its heads read."""
    kind = {"k": S_K, "v": S_V, "kslow": S_KSLOW, "vslow": S_VSLOW}[which]
    n = num_pages * sp.page * sp.D
    flat = None if out is None else out.reshape(-1)
    return normal_bf16(sp.seed, stream_id(kind), n, out=flat).reshape(
        num_pages, sp.page, sp.D)


def pool_page_bits(sp: Spec, which: str, pages: np.ndarray) -> np.ndarray:
    """Contents of selected physical pages only (same values as pool_bits), for sampled
    checks at full size: uint16[len(pages), page, D]."""
    kind = {"k": S_K, "v": S_V, "kslow": S_KSLOW, "vslow": S_VSLOW}[which]
    per = sp.page * sp.D
    out = np.empty((len(pages), sp.page, sp.D), dtype=np.uint16)
    for i, p in enumerate(np.asarray(pages, dtype=np.int64)):
        normal_bf16(sp.seed, stream_id(kind), per, i0=int(p) * per,
                    out=out[i].reshape(-1))
    return out


# ---------------------------------------------------------------------------------------
# Decode-step write path inputs.
# ---------------------------------------------------------------------------------------

def new_kv_bits(sp: Spec, step: int, which: str, layer: int = 0) -> np.ndarray:
    """K or V row of the token appended at decode step `step`, per (sequence, KV head):
    bf16 bits uint16[B, Hkv, D], N(0, 1)."""
    kind = {"k": S_NEWK, "v": S_NEWV}[which]
    n = sp.B * sp.Hkv * sp.D
    return normal_bf16(sp.seed, stream_id(kind, (layer << 16) | step), n).reshape(sp.B, sp.Hkv, sp.D)


def init_scores(sp: Spec, n: int, layer: int = 0) -> np.ndarray:
    """n accumulated attention scores float32 in [0, 4), 24-bit resolution (exact in fp32)."""
    d = draws(sp.seed, stream_id(S_SCORE, layer), n)
    return ((d >> np.uint64(40)).astype(np.float64) * 2.0 ** -22).astype(np.float32)


def retained_positions(sp: Spec, kv_len: np.ndarray, seen: np.ndarray, recent: int,
                       layer: int = 0) -> list:
    """Admission state of each head for the score-based policy: the positions its kv_len
    retained slots hold, given `seen` tokens so far. The last min(recent, kv_len) positions
    are kept and the rest is a seeded choice among the older ones; slots hold them in
    increasing position order. Returns one int32 array per (b, h), row-major."""
    out = []
    kv = np.asarray(kv_len).reshape(-1)
    sn = np.asarray(seen).reshape(-1)
    for i in range(kv.size):
        n, L = int(kv[i]), int(sn[i])
        r = min(recent, n, L)
        older = L - r
        k = min(n - r, older)
        pick = permutation(sp.seed, stream_id(S_PICK, (layer << 20) | i), older)[:k] if k > 0 else \
            np.zeros(0, np.int64)
        pos = np.concatenate([np.sort(pick.astype(np.int64)), np.arange(L - r, L)]).astype(np.int32)
        out.append(pos)
    return out
