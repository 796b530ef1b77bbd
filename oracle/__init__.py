"""CPU oracle for ragged / prefix-shared / tiered paged decode attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg and reference arm may import this package. The product (``non_uniform_paged_flash_b200``) never
imports it, and the two share no code.

The arithmetic lives in ``tg_oracle.c`` (plain loops, fp64 attention); this module only
compiles it and marshals numpy arrays. Each function cites, in the C source, the passage of
the source pages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tg_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile tg_oracle.c (gcc -O2, OpenMP, strict IEEE float: no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        p, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.or_num_threads.restype = ctypes.c_int
        lib.or_retained_lengths.argtypes = [i64, p, p, p]
        lib.or_budget_groups.argtypes = [i32, p, i32, p]
        lib.or_reservation_layout.restype = i64
        lib.or_reservation_layout.argtypes = [i64, p, i32, i32, i32, p, i32, i32, p, p, p, p, p]
        lib.or_group_tables.restype = i64
        lib.or_group_tables.argtypes = [i32, i32, p, i32, p, p, p, p, p]
        lib.or_decode.restype = ctypes.c_int
        lib.or_decode.argtypes = [i32, i32, i32, i32, i32, p, p, p, i64, p, p, p, p, p, f64,
                                  i64, p, p, p]
        lib.or_tiered_decode.restype = ctypes.c_int
        lib.or_tiered_decode.argtypes = [i32, i32, i32, i32, i32, p, p, p, p, p, i64, p, p,
                                         p, p, i64, p, p, p, p, f64, i64, p, p, p]
        lib.or_quantize_int8.argtypes = [i64, i32, p, p, p]
        lib.or_quantize_int4.argtypes = [i64, i32, p, p, p]
        lib.or_unpack_int4.argtypes = [i64, i32, p, p]
        lib.or_lse_merge.argtypes = [i32, i64, i32, p, p, p, p]
        lib.or_place_sequences.argtypes = [i32, p, i32, p]
        lib.or_sink_recent_slot.argtypes = [i32, i32, i32, p]
        lib.or_sink_recent_slot.restype = i32
        lib.or_h2o_victim.argtypes = [i32, i32, i32, p, p, i32]
        lib.or_h2o_victim.restype = i32
        lib.or_token_scores.argtypes = [i32, i32, i32, i32, i32, p, p, i64, p, p, p, f64, p]
        lib.or_token_scores.restype = ctypes.c_int
        lib.or_h2o_accumulate.argtypes = [i32, i32, p, p, p, p]
        lib.or_tier_step.argtypes = [i32, i32, i32, i32, p, p]
        lib.or_tier_step.restype = ctypes.c_int
        lib.or_splitzip_codebook.argtypes = [i64, p, p]
        lib.or_splitzip_encode.argtypes = [i64, p, p, p, p, p, p]
        lib.or_splitzip_encode.restype = i64
        lib.or_splitzip_decode.argtypes = [i64, p, p, p, i64, p, p, p]
        _lib = lib
    return _lib


def _c(a, dtype):
    """Contiguous array of dtype (no copy when already so)."""
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data


def num_threads() -> int:
    return int(_L().or_num_threads())


def retained_lengths(full_len, ratio_ppm) -> np.ndarray:
    L = _c(full_len, np.int32)
    r = _c(ratio_ppm, np.int32)
    assert L.shape == r.shape
    out = np.empty(L.shape, dtype=np.int32)
    _L().or_retained_lengths(L.size, _ptr(L), _ptr(r), _ptr(out))
    return out


def budget_groups(budget_ppm, n_groups: int) -> np.ndarray:
    b = _c(budget_ppm, np.int32).reshape(-1)
    out = np.empty(b.size, dtype=np.int32)
    _L().or_budget_groups(b.size, _ptr(b), n_groups, _ptr(out))
    return out


def reservation_layout(num_pages, free_order, page, kv_len, seg_tokens=(), chain=None):
    """Pages of every (sequence, head) under Budget Reservation from a FIFO free list.

    kv_len int[B, Hkv]; seg_tokens: shared segment sizes; chain int[B, chain_len] segment ids.
    Returns (page_ids flat, head_count int32[B, Hkv], seg_pages flat)."""
    kv = _c(kv_len, np.int32)
    B, Hkv = kv.shape
    fo = _c(free_order, np.int32)
    seg = _c(np.asarray(seg_tokens, dtype=np.int32).reshape(-1), np.int32)
    ch = _c(np.zeros((B, 0), np.int32) if chain is None else chain, np.int32)
    chain_len = ch.shape[1] if ch.ndim == 2 else 0
    cap = int(kv.astype(np.int64).sum() // page + 2 * B * Hkv + 8)
    ids = np.empty(cap, dtype=np.int32)
    cnt = np.empty((B, Hkv), dtype=np.int32)
    segp = np.empty(max(1, int(sum(Hkv * (s // page) for s in seg))), dtype=np.int32)
    w = _L().or_reservation_layout(num_pages, _ptr(fo), page, Hkv, seg.size, _ptr(seg), B,
                                   chain_len, _ptr(ch), _ptr(kv), _ptr(ids), _ptr(cnt),
                                   _ptr(segp))
    if w < 0:
        raise RuntimeError({-1: "pool exhausted", -2: "head shorter than its shared prefix"}[w])
    nseg = int(sum(Hkv * (s // page) for s in seg))
    return ids[:w].copy(), cnt, segp[:nseg].copy()


def group_tables(group_of_head, n_groups, page_ids, head_count):
    """Concatenated per-group dense page tables. Returns (table, head_off[B, Hkv], group_off)."""
    cnt = _c(head_count, np.int32)
    B, Hkv = cnt.shape
    goh = _c(group_of_head, np.int32)
    ids = _c(page_ids, np.int32)
    cap = 0
    for g in range(n_groups):
        hs = [h for h in range(Hkv) if goh[h] == g]
        if hs and B > 0:
            cap += B * len(hs) * int(cnt[:, hs].max())
    table = np.empty(max(cap, 1), dtype=np.int32)
    off = np.empty((B, Hkv), dtype=np.int64)
    goff = np.empty(n_groups + 1, dtype=np.int64)
    n = _L().or_group_tables(B, Hkv, _ptr(goh), n_groups, _ptr(ids), _ptr(cnt), _ptr(table),
                             _ptr(off), _ptr(goff))
    return table[:n].copy(), off, goff


def decode(q_bits, k_bits, v_bits, table, head_off, kv_len, scale, tok_lo=None, tok_hi=None,
           sel=None):
    """fp64 paged decode attention. q_bits uint16[B, Hq, D]; pools uint16[P, page, D].
    Returns (out float64[rows, D], lse float64[rows]); rows = B*Hq or len(sel)."""
    q = _c(q_bits, np.uint16)
    B, Hq, D = q.shape
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    P, page, D2 = k.shape
    assert D2 == D and v.shape == k.shape
    kv = _c(kv_len, np.int32)
    Hkv = kv.shape[1]
    t = _c(table, np.int32)
    off = _c(head_off, np.int64)
    lo = None if tok_lo is None else _c(tok_lo, np.int32)
    hi = None if tok_hi is None else _c(tok_hi, np.int32)
    s = None if sel is None else _c(sel, np.int64)
    rows = B * Hq if s is None else s.size
    out = np.empty((rows, D), dtype=np.float64)
    lse = np.empty(rows, dtype=np.float64)
    e = _L().or_decode(B, Hq, Hkv, D, page, _ptr(q), _ptr(k), _ptr(v), P, _ptr(t), _ptr(off),
                       _ptr(kv), _ptr(lo), _ptr(hi), float(scale), -1 if s is None else s.size,
                       _ptr(s), _ptr(out), _ptr(lse))
    if e:
        raise RuntimeError(f"oracle decode error {e}")
    return out, lse


def tiered_decode(q_bits, k_q8, v_q8, k_scale, v_scale, slow_table, slow_off, k_fast_bits,
                  v_fast_bits, fast_table, fast_off, kv_len, fast_len, scale, sel=None):
    """fp64 tiered decode. Slow pools int8[Ps, page, D] + float32[Ps, page] scales; fast pools
    bf16 bits uint16[Pf, page, D]."""
    q = _c(q_bits, np.uint16)
    B, Hq, D = q.shape
    kq, vq = _c(k_q8, np.int8), _c(v_q8, np.int8)
    ks, vs = _c(k_scale, np.float32), _c(v_scale, np.float32)
    kf, vf = _c(k_fast_bits, np.uint16), _c(v_fast_bits, np.uint16)
    Ps, page, _ = kq.shape
    Pf = kf.shape[0]
    kv = _c(kv_len, np.int32)
    fl = _c(fast_len, np.int32)
    Hkv = kv.shape[1]
    st, so = _c(slow_table, np.int32), _c(slow_off, np.int64)
    ft, fo = _c(fast_table, np.int32), _c(fast_off, np.int64)
    s = None if sel is None else _c(sel, np.int64)
    rows = B * Hq if s is None else s.size
    out = np.empty((rows, D), dtype=np.float64)
    lse = np.empty(rows, dtype=np.float64)
    e = _L().or_tiered_decode(B, Hq, Hkv, D, page, _ptr(q), _ptr(kq), _ptr(vq), _ptr(ks),
                              _ptr(vs), Ps, _ptr(st), _ptr(so), _ptr(kf), _ptr(vf), Pf,
                              _ptr(ft), _ptr(fo), _ptr(kv), _ptr(fl), float(scale),
                              -1 if s is None else s.size, _ptr(s), _ptr(out), _ptr(lse))
    if e:
        raise RuntimeError(f"oracle tiered decode error {e}")
    return out, lse


def quantize_int8(src_bits):
    """Per-row symmetric absmax INT8 of bf16 rows. src uint16[..., D] ->
    (codes int8[..., D], scale float32[...])."""
    a = _c(src_bits, np.uint16)
    D = a.shape[-1]
    rows = a.size // D
    codes = np.empty(a.shape, dtype=np.int8)
    scale = np.empty(a.shape[:-1], dtype=np.float32)
    _L().or_quantize_int8(rows, D, _ptr(a), _ptr(codes), _ptr(scale))
    return codes, scale


def quantize_int4(src_bits):
    """Per-row symmetric absmax INT4 of bf16 rows, packed two codes per byte (byte i: d = i low
    nibble, d = i + D/2 high nibble, offset-binary code + 8). src uint16[..., D] ->
    (packed uint8[..., D/2], scale float32[...])."""
    a = _c(src_bits, np.uint16)
    D = a.shape[-1]
    if D % 2:
        raise ValueError("INT4 rows need an even D")
    rows = a.size // D
    packed = np.empty(a.shape[:-1] + (D // 2,), dtype=np.uint8)
    scale = np.empty(a.shape[:-1], dtype=np.float32)
    _L().or_quantize_int4(rows, D, _ptr(a), _ptr(packed), _ptr(scale))
    return packed, scale


def unpack_int4(packed):
    """Codes int8[..., D] of packed INT4 rows uint8[..., D/2]."""
    a = _c(packed, np.uint8)
    D = 2 * a.shape[-1]
    rows = a.size // (D // 2)
    codes = np.empty(a.shape[:-1] + (D,), dtype=np.int8)
    _L().or_unpack_int4(rows, D, _ptr(a), _ptr(codes))
    return codes


def lse_merge(parts_o, parts_lse):
    """parts_o float64[S, rows, D], parts_lse float64[S, rows] -> (out[rows, D], lse[rows])."""
    po = _c(parts_o, np.float64)
    pl = _c(parts_lse, np.float64)
    S, rows, D = po.shape
    out = np.empty((rows, D), dtype=np.float64)
    lse = np.empty(rows, dtype=np.float64)
    _L().or_lse_merge(S, rows, D, _ptr(po), _ptr(pl), _ptr(out), _ptr(lse))
    return out, lse


def place_sequences(seq_bytes, n_gpus: int) -> np.ndarray:
    b = _c(seq_bytes, np.int64)
    out = np.empty(b.size, dtype=np.int32)
    _L().or_place_sequences(b.size, _ptr(b), n_gpus, _ptr(out))
    return out


# ---------------------------------------------------------------------------------------
# Decode-step write path.
# ---------------------------------------------------------------------------------------

def sink_recent_slot(budget: int, sink: int, kv_len: int, slot_pos) -> int:
    """Slot that receives a head's new token under the sink + recent rule (or -1)."""
    sp = _c(slot_pos, np.int32)
    return int(_L().or_sink_recent_slot(int(budget), int(sink), int(kv_len), _ptr(sp)))


def h2o_victim(budget: int, recent: int, kv_len: int, slot_pos, score, new_pos: int) -> int:
    """Slot that receives a head's new token under the H2O rule (or -1)."""
    sp = _c(slot_pos, np.int32)
    sc = _c(score, np.float32)
    return int(_L().or_h2o_victim(int(budget), int(recent), int(kv_len), _ptr(sp), _ptr(sc),
                                  int(new_pos)))


def token_scores(q_bits, k_bits, table, head_off, kv_len, scale, table_len: int, page: int = 16):
    """Per-token scores of every retained token, float64[table_len * page, G]; NaN where no
    token is retained."""
    q = _c(q_bits, np.uint16)
    k = _c(k_bits, np.uint16)
    B, Hq, D = q.shape
    kl = _c(kv_len, np.int32)
    Hkv = kl.size // B
    G = Hq // Hkv
    out = np.full((int(table_len) * page, G), np.nan, dtype=np.float64)
    rc = _L().or_token_scores(B, Hq, Hkv, D, page, _ptr(q), _ptr(k), k.shape[0],
                              _ptr(_c(table, np.int32)), _ptr(_c(head_off, np.int64)), _ptr(kl),
                              float(scale), _ptr(out))
    if rc:
        raise ValueError(f"or_token_scores failed ({rc})")
    return out


def h2o_accumulate(s, lse, score):
    """score[t] + sum_g exp(s[t, g] - lse[g]) for one head, float32[n]."""
    s_ = _c(s, np.float64)
    n, G = s_.shape
    l_ = _c(lse, np.float64)
    sc = _c(score, np.float32)
    out = np.empty(n, dtype=np.float32)
    _L().or_h2o_accumulate(n, G, _ptr(s_), _ptr(l_), _ptr(sc), _ptr(out))
    return out


def tier_step(n: int, f: int, cap: int, slow_cap: int):
    """(fast slot, slow index) of appending position n to a head with f fast tokens out of n;
    slow index -1 when nothing moves; (-1, -1) when the state is outside the rules."""
    fs = np.zeros(1, np.int32)
    si = np.zeros(1, np.int32)
    rc = _L().or_tier_step(int(n), int(f), int(cap), int(slow_cap), _ptr(fs), _ptr(si))
    return (int(fs[0]), int(si[0])) if rc == 0 else (-1, -1)


def splitzip_encode(x_bits):
    """bf16 bits -> (codebook uint8[16], sm uint8[n], codes uint8[(n+1)//2], esc_pos int64[k],
    esc_exp uint8[k])."""
    x = _c(x_bits, np.uint16).reshape(-1)
    n = x.size
    cb = np.empty(16, np.uint8)
    _L().or_splitzip_codebook(n, _ptr(x), _ptr(cb))
    sm = np.empty(max(n, 1), np.uint8)
    codes = np.empty(max((n + 1) // 2, 1), np.uint8)
    pos = np.empty(max(n, 1), np.int64)
    exp = np.empty(max(n, 1), np.uint8)
    k = int(_L().or_splitzip_encode(n, _ptr(x), _ptr(cb), _ptr(sm), _ptr(codes), _ptr(pos), _ptr(exp)))
    return cb, sm[:n], codes[:(n + 1) // 2], pos[:k], exp[:k]


def splitzip_decode(n, codebook, sm, codes, esc_pos, esc_exp):
    out = np.empty(max(int(n), 1), np.uint16)
    cb, s_, c_ = _c(codebook, np.uint8), _c(sm, np.uint8), _c(codes, np.uint8)
    p_, e_ = _c(esc_pos, np.int64), _c(esc_exp, np.uint8)
    _L().or_splitzip_decode(int(n), _ptr(cb), _ptr(s_), _ptr(c_), p_.size, _ptr(p_), _ptr(e_), _ptr(out))
    return out[:int(n)]
