"""Python binding of libtg, the B200 ragged / prefix-shared / tiered paged decode library.

Argument marshalling only: every step runs in libtg.so (host C++ for admission-time steps,
sm_100a CUDA kernels for the decode). There is no fallback: if libtg.so is missing or fails
to load, importing the library raises. The C ABI is declared in include/tg.h; each function
here has the same name and documents only how Python arguments map onto it.

Host arrays are numpy arrays (converted to contiguous arrays of the ABI's dtype). Device
arrays are CUDA tensors (anything with .data_ptr()); the stream defaults to torch's current
stream on the current device.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtg.so")

TG_OK, TG_EINVAL, TG_ENOSPC, TG_EBADPAGE, TG_ECUDA, TG_ETIMEOUT = 0, 1, 2, 3, 4, 5
TG_ENOMEM, TG_ENOTFOUND, TG_EUNSUPPORTED, TG_EEXIST = 6, 7, 8, 9
TG_MAX_HEAD_TOKENS = 1 << 30   # longest retained length of one (sequence, KV head) a plan accepts


class TGError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib().tg_strerror(status).decode()
        if status == TG_ECUDA:
            msg += " — " + _lib().tg_last_cuda_error().decode()
        super().__init__(f"{where}: {msg} (status {status})")


class tg_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("D", ctypes.c_int32), ("page", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("num_pages", ctypes.c_int64), ("num_slow_pages", ctypes.c_int64)]


class tg_plan_opts(ctypes.Structure):
    _fields_ = [("num_workers", ctypes.c_int32), ("min_splits", ctypes.c_int32),
                ("max_chunk_pages", ctypes.c_int32), ("host_only", ctypes.c_int32),
                ("device", ctypes.c_int32), ("static_permille", ctypes.c_int32),
                ("dyn_chunk_pages", ctypes.c_int32), ("early_prologue", ctypes.c_int32),
                ("wait_limit_us", ctypes.c_int32), ("test_withhold_page", ctypes.c_int32),
                ("capacity", ctypes.c_int32),
                ("out_f32", ctypes.c_int32), ("slow_bits", ctypes.c_int32),
                ("whole_heads", ctypes.c_int32)]


class tg_plan_info(ctypes.Structure):
    _fields_ = [("n_items", ctypes.c_int64), ("n_partials", ctypes.c_int64),
                ("n_merge", ctypes.c_int64), ("n_empty", ctypes.c_int64),
                ("n_dynamic", ctypes.c_int64),
                ("n_workers", ctypes.c_int32),
                ("grid", ctypes.c_int32), ("block", ctypes.c_int32),
                ("smem_bytes", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("n_cascade", ctypes.c_int32), ("device_bytes", ctypes.c_int64),
                ("kv_bytes", ctypes.c_int64)]


_L = None

#: Query rows of one prefix-cascade unit (two tensor-core tiles of 128 rows).
CASCADE_ROWS = 256

# (name, restype, argtypes)
_P, _I32, _I64, _F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
_SIGS = [
    ("tg_strerror", ctypes.c_char_p, [ctypes.c_int]),
    ("tg_last_cuda_error", ctypes.c_char_p, []),
    ("tg_retained_lengths", ctypes.c_int, [_I64, _P, _P, _P]),
    ("tg_budget_groups", ctypes.c_int, [_I32, _P, _I32, _P]),
    ("tg_alloc_create", ctypes.c_int, [_I64, _I32, ctypes.c_uint64, ctypes.POINTER(_P)]),
    ("tg_alloc_create_ordered", ctypes.c_int, [_I64, _I32, _P, ctypes.POINTER(_P)]),
    ("tg_alloc_destroy", None, [_P]),
    ("tg_alloc_free_pages", _I64, [_P]),
    ("tg_alloc_refcount", _I32, [_P, _I32]),
    ("tg_share_segment", ctypes.c_int, [_P, _I32, _I32, _P, _P]),
    ("tg_reserve", ctypes.c_int, [_P, _I32, _I32, _P, _I32, _P, _P, _I64, _P, _P]),
    ("tg_release", ctypes.c_int, [_P, _I32]),
    ("tg_release_segment", ctypes.c_int, [_P, _I32]),
    ("tg_build_group_tables", ctypes.c_int, [_I32, _I32, _P, _P, _I32, _P, _P, _P, _P]),
    ("tg_place_sequences", ctypes.c_int, [_I32, _P, _I32, _P]),
    ("tg_plan_create", ctypes.c_int, [ctypes.POINTER(tg_shape), _P, _P, _P, _P, _I32, _I64,
                                      ctypes.POINTER(tg_plan_opts), ctypes.POINTER(_P)]),
    ("tg_plan_destroy", None, [_P]),
    ("tg_plan_get_info", ctypes.c_int, [_P, ctypes.POINTER(tg_plan_info)]),
    ("tg_plan_items", ctypes.c_int, [_P, _P]),
    ("tg_plan_status", ctypes.c_int, [_P, _P]),
    ("tg_plan_timing_enable", ctypes.c_int, [_P, _I32]),
    ("tg_plan_timing_read", ctypes.c_int, [_P, _P, _P, _P]),
    ("tg_plan_trace_enable", ctypes.c_int, [_P, _I32]),
    ("tg_plan_trace_read", ctypes.c_int, [_P, _P, _P]),
    ("tg_ragged_paged_decode", ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _F32, _P, _P, _P]),
    ("tg_ragged_paged_decode_noalloc", ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _F32, _P,
                                                      _P, _P]),
    ("tg_ragged_paged_decode_noalloc_status", ctypes.c_int, [_P]),
    ("tg_tiered_decode", ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                        _F32, _P, _P, _P]),
    ("tg_lse_merge", ctypes.c_int, [_I64, _I32, _P, _P, _P, _P, _P, _P]),
    ("tg_quantize_int8", ctypes.c_int, [_I64, _I32, _P, _P, _P, _P]),
    ("tg_quantize_int4", ctypes.c_int, [_I64, _I32, _P, _P, _P, _P]),
    ("tg_ragged_paged_decode_scores", ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _F32, _P,
                                                     _P, _P, _P]),
    ("tg_append_sink_recent", ctypes.c_int, [ctypes.POINTER(tg_shape), _I32, _P, _P, _P, _P, _P,
                                             _P, _P, _P, _P, _P, _P]),
    ("tg_append_h2o", ctypes.c_int, [ctypes.POINTER(tg_shape), _P, _P, _P, _P, _P, _P, _P, _P,
                                     _P, _P, _P, _P, _P, _P]),
    ("tg_h2o_update", ctypes.c_int, [ctypes.POINTER(tg_shape), _I32, _P, _P, _P, _P, _P, _P, _P,
                                     _P, _P, _P]),
    ("tg_plan_create_cascade", ctypes.c_int, [ctypes.POINTER(tg_shape), _P, _P, _P, _I32, _P, _P,
                                              _I64, _I32, ctypes.POINTER(tg_plan_opts),
                                              ctypes.POINTER(_P)]),
    ("tg_plan_cascade_units", ctypes.c_int, [_P, _P]),
    ("tg_tiered_append", ctypes.c_int, [ctypes.POINTER(tg_shape), _P, _P, _P, _P, _P, _P, _P, _P,
                                        _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    ("tg_tiered_append_int4", ctypes.c_int, [ctypes.POINTER(tg_shape), _P, _P, _P, _P, _P, _P, _P,
                                             _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    ("tg_splitzip_workspace_bytes", _I64, [_I64]),
    ("tg_splitzip_encode", ctypes.c_int, [_I64, _P, _P, _P, _P, _P, _P, _I64, _P, _P, _P]),
    ("tg_splitzip_decode", ctypes.c_int, [_I64, _P, _P, _P, _P, _P, _P, _I64, _P, _P]),
    ("tg_host_pipe_create", ctypes.c_int, [_P, ctypes.POINTER(_P)]),
    ("tg_host_pipe_destroy", None, [_P]),
    ("tg_host_pipe_wait", ctypes.c_int, [_P]),
    ("tg_host_pipe_after", ctypes.c_int, [_P, _P]),
    ("tg_host_pipe_join", ctypes.c_int, [_P, _P]),
    ("tg_ragged_paged_decode_host", ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _F32, _P,
                                                   _P, _P]),
    ("tg_tiered_decode_host", ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                             _P, _P, _F32, _P, _P, _P]),
    ("tg_slow_stream_create", ctypes.c_int, [ctypes.POINTER(tg_shape), _P, _P, _P, _P, _I32, _P, _P,
                                             _I64, _I32, _I32, ctypes.POINTER(tg_plan_opts),
                                             ctypes.POINTER(_P)]),
    ("tg_slow_stream_destroy", None, [_P]),
    ("tg_slow_stream_blocks", ctypes.c_int, [_P, _P, _P, _P]),
    ("tg_slow_stream_status", ctypes.c_int, [_P, _P]),
    ("tg_tiered_decode_streamed", ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _F32,
                                                 _P, _P, _P]),
]

#: Symbols the C ABI exports (include/tg.h).
ABI_SYMBOLS = tuple(n for n, _, _ in _SIGS)


def _lib():
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libtg.so not built ({LIB_PATH}); run "
                              "`python -m non_uniform_paged_flash_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, res, args in _SIGS:
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _L = lib
    return _L


def load():
    """Load libtg.so (raises if it is missing)."""
    return _lib()


def _check(status: int, where: str):
    if status != TG_OK:
        raise TGError(status, where)


def _h(a, dtype):
    """Host array as a contiguous numpy array of dtype."""
    return np.ascontiguousarray(a, dtype=dtype)


def _hp(a):
    return None if a is None else a.ctypes.data


def _count(a, n, what, at_least=False):
    """A host array holds n entries (at least n with at_least): the C side reads that many."""
    if a is None:
        return
    if (a.size < n) if at_least else (a.size != n):
        raise ValueError(f"{what}: {a.size} entries, {'at least ' if at_least else ''}{n} expected")


def _dp(t):
    """Device pointer of a CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not getattr(t, "is_cuda", False):
        raise ValueError("expected a CUDA tensor for a device argument")
    return t.data_ptr()


def _need(t, n, dtype, what):
    """A tensor argument holds at least n elements of dtype (the C ABI takes bare pointers)."""
    import torch
    if t is None:
        raise ValueError(f"{what}: missing")
    if t.dtype != dtype:
        raise ValueError(f"{what}: expected {dtype}, got {t.dtype}")
    if t.numel() < n:
        raise ValueError(f"{what}: {t.numel()} elements, the plan needs {n}")
    if not t.is_contiguous():
        raise ValueError(f"{what}: must be contiguous")


def _check_io(plan, q, out, lse):
    """q bf16 [B][Hq][D]; out bf16 (fp32 for out_f32 plans) [B][Hq][D]; lse fp32 [B][Hq]."""
    import torch
    s = plan.shape
    rows = s.B * s.Hq
    _need(q, rows * s.D, torch.bfloat16, "q")
    _need(out, rows * s.D, torch.float32 if plan.out_f32 else torch.bfloat16, "out")
    _need(lse, rows, torch.float32, "lse")


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


# ------------------------------------------------------------------------------------------
# Host-side admission steps
# ------------------------------------------------------------------------------------------

def tg_retained_lengths(full_len, ratio_ppm) -> np.ndarray:
    L = _h(full_len, np.int32)
    r = _h(ratio_ppm, np.int32)
    if L.shape != r.shape:
        raise ValueError("shape mismatch")
    out = np.empty(L.shape, dtype=np.int32)
    _check(_lib().tg_retained_lengths(L.size, _hp(L), _hp(r), _hp(out)), "tg_retained_lengths")
    return out


def tg_budget_groups(budget_ppm, n_groups: int) -> np.ndarray:
    b = _h(budget_ppm, np.int32).reshape(-1)
    out = np.empty(b.size, dtype=np.int32)
    _check(_lib().tg_budget_groups(b.size, _hp(b), n_groups, _hp(out)), "tg_budget_groups")
    return out


def tg_alloc_create(num_pages: int, page: int = 16, seed: int = 0):
    """Allocator whose initial free list is the library's seeded shuffle of the page ids."""
    h = ctypes.c_void_p()
    _check(_lib().tg_alloc_create(num_pages, page, ctypes.c_uint64(int(seed) & (2**64 - 1)),
                                  ctypes.byref(h)), "tg_alloc_create")
    h.page = page   # output buffers of the calls below are sized with the allocator's page
    return h


def tg_alloc_create_ordered(num_pages: int, page: int = 16, free_order=None):
    fo = None if free_order is None else _h(free_order, np.int32).reshape(-1)
    _count(fo, num_pages, "free_order")
    h = ctypes.c_void_p()
    _check(_lib().tg_alloc_create_ordered(num_pages, page, _hp(fo), ctypes.byref(h)),
           "tg_alloc_create_ordered")
    h.page = page   # output buffers of the calls below are sized with the allocator's page
    return h


def _alloc_page(a, page):
    """The allocator's page size (a page argument that disagrees with it is refused)."""
    own = getattr(a, "page", None)
    if own is None:
        return page
    if page is not None and page != own:
        raise ValueError(f"page {page} given, the allocator's page is {own}")
    return own


def tg_alloc_destroy(a):
    _lib().tg_alloc_destroy(a)


def tg_alloc_free_pages(a) -> int:
    return int(_lib().tg_alloc_free_pages(a))


def tg_alloc_refcount(a, page_id: int) -> int:
    return int(_lib().tg_alloc_refcount(a, page_id))


def tg_share_segment(a, n_tokens: int, n_heads: int, page: int = None):
    """Returns (seg_id, page_ids int32[n_heads, n_tokens // page])."""
    page = _alloc_page(a, page)
    if page is None:
        raise ValueError("page size unknown: pass the allocator's page")
    full = n_tokens // page
    ids = np.empty((n_heads, full), dtype=np.int32)
    sid = ctypes.c_int32()
    _check(_lib().tg_share_segment(a, n_tokens, n_heads, ctypes.byref(sid), _hp(ids)),
           "tg_share_segment")
    return sid.value, ids


def tg_reserve(a, seq_id: int, kv_len, prefix_segs=(), page: int = None,
               with_counts: bool = False):
    """Reserve all heads of one sequence; returns its page ids (flat, head after head), and
    with with_counts also each head's page count (int32[n_heads])."""
    page = _alloc_page(a, page) or 1   # page 1 sizes the buffer for any allocator
    kv = _h(kv_len, np.int32).reshape(-1)
    segs = _h(np.asarray(prefix_segs, dtype=np.int32).reshape(-1), np.int32)
    cap = int(kv.astype(np.int64).sum() // page + kv.size * (1 + max(1, segs.size)))
    ids = np.empty(cap, dtype=np.int32)
    counts = np.empty(kv.size, dtype=np.int32)
    n = ctypes.c_int64()
    _check(_lib().tg_reserve(a, seq_id, kv.size, _hp(kv), segs.size,
                             _hp(segs) if segs.size else None, _hp(ids), cap, _hp(counts),
                             ctypes.byref(n)), "tg_reserve")
    ids = ids[:n.value].copy()
    return (ids, counts) if with_counts else ids


def tg_release(a, seq_id: int):
    _check(_lib().tg_release(a, seq_id), "tg_release")


def tg_release_segment(a, seg_id: int):
    _check(_lib().tg_release_segment(a, seg_id), "tg_release_segment")


def tg_build_group_tables(head_count, group_of_head, n_groups: int, page_ids):
    """Returns (table int32[len], head_off int64[B, Hkv], group_off int64[n_groups + 1])."""
    hc = _h(head_count, np.int32)
    B, Hkv = hc.shape
    goh = _h(group_of_head, np.int32).reshape(-1)
    ids = _h(page_ids, np.int32).reshape(-1)
    _count(goh, Hkv, "group_of_head")
    _count(ids, int(np.maximum(hc, 0).astype(np.int64).sum()), "page_ids", at_least=True)
    goff = np.empty(n_groups + 1, dtype=np.int64)
    _check(_lib().tg_build_group_tables(B, Hkv, _hp(hc), _hp(goh), n_groups, None, None, None,
                                        _hp(goff)), "tg_build_group_tables")
    table = np.empty(max(1, int(goff[-1])), dtype=np.int32)
    off = np.empty((B, Hkv), dtype=np.int64)
    _check(_lib().tg_build_group_tables(B, Hkv, _hp(hc), _hp(goh), n_groups, _hp(ids),
                                        _hp(table), _hp(off), _hp(goff)), "tg_build_group_tables")
    return table[:int(goff[-1])].copy(), off, goff


def tg_place_sequences(seq_bytes, n_gpus: int) -> np.ndarray:
    b = _h(seq_bytes, np.int64)
    out = np.empty(b.size, dtype=np.int32)
    _check(_lib().tg_place_sequences(b.size, _hp(b), n_gpus, _hp(out)), "tg_place_sequences")
    return out


# ------------------------------------------------------------------------------------------
# Plan
# ------------------------------------------------------------------------------------------

@dataclass
class Plan:
    """Owns a tg_plan handle; destroy() (or garbage collection) frees it."""
    handle: ctypes.c_void_p
    shape: tg_shape
    tiered: bool
    out_f32: bool = False

    def destroy(self):
        if self.handle:
            _lib().tg_plan_destroy(self.handle)
            self.handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def make_shape(B, Hq, Hkv, D, num_pages, num_slow_pages=0, page=16) -> tg_shape:
    return tg_shape(B, Hq, Hkv, D, page, 0, num_pages, num_slow_pages)


def tg_plan_create(shape: tg_shape, kv_len, group_of_head, group_off, fast_len=None,
                   slow_table_len: int = 0, num_workers: int = 0, min_splits: int = 1,
                   max_chunk_pages: int = 0, host_only: bool = False, device: int = -1,
                   static_permille: int = 0, dyn_chunk_pages: int = 0,
                   early_prologue: bool = False, wait_limit_us: int = 0,
                   test_withhold_page: int = 0, capacity: bool = False,
                   out_f32: bool = False, slow_bits: int = 8, whole_heads: bool = False) -> Plan:
    kv = _h(kv_len, np.int32).reshape(-1)
    fl = None if fast_len is None else _h(fast_len, np.int32).reshape(-1)
    goh = _h(group_of_head, np.int32).reshape(-1)
    goff = _h(group_off, np.int64).reshape(-1)
    _count(kv, shape.B * shape.Hkv, "kv_len")
    _count(fl, shape.B * shape.Hkv, "fast_len")
    _count(goh, shape.Hkv, "group_of_head")
    _count(goff, 2, "group_off", at_least=True)
    opts = tg_plan_opts(num_workers, min_splits, max_chunk_pages, int(host_only), device,
                        static_permille, dyn_chunk_pages, int(early_prologue), wait_limit_us,
                        test_withhold_page, int(capacity), int(out_f32), int(slow_bits),
                        int(whole_heads))
    h = ctypes.c_void_p()
    _check(_lib().tg_plan_create(ctypes.byref(shape), _hp(kv), _hp(fl), _hp(goh), _hp(goff),
                                 goff.size - 1, slow_table_len, ctypes.byref(opts),
                                 ctypes.byref(h)), "tg_plan_create")
    return Plan(h, shape, fl is not None, bool(out_f32))


def tg_plan_create_cascade(shape: tg_shape, kv_len, group_of_head, group_off, page_table,
                           head_page_off, min_readers: int = 2, num_workers: int = 0,
                           min_splits: int = 1, max_chunk_pages: int = 0, host_only: bool = False,
                           device: int = -1, static_permille: int = 0, dyn_chunk_pages: int = 0,
                           early_prologue: bool = False, wait_limit_us: int = 0,
                           out_f32: bool = False) -> Plan:
    """Prefix-aware cascade plan from the host page table (see include/tg.h)."""
    kv = _h(kv_len, np.int32).reshape(-1)
    goh = _h(group_of_head, np.int32).reshape(-1)
    goff = _h(group_off, np.int64).reshape(-1)
    tbl = _h(page_table, np.int32).reshape(-1)
    hoff = _h(head_page_off, np.int64).reshape(-1)
    _count(kv, shape.B * shape.Hkv, "kv_len")
    _count(goh, shape.Hkv, "group_of_head")
    _count(goff, 2, "group_off", at_least=True)
    _count(hoff, shape.B * shape.Hkv, "head_page_off")
    opts = tg_plan_opts(num_workers, min_splits, max_chunk_pages, int(host_only), device,
                        static_permille, dyn_chunk_pages, int(early_prologue), wait_limit_us, 0, 0,
                        int(out_f32), 8)
    h = ctypes.c_void_p()
    _check(_lib().tg_plan_create_cascade(ctypes.byref(shape), _hp(kv), _hp(goh), _hp(goff),
                                         goff.size - 1, _hp(tbl), _hp(hoff), tbl.size,
                                         int(min_readers), ctypes.byref(opts), ctypes.byref(h)),
           "tg_plan_create_cascade")
    return Plan(h, shape, False, bool(out_f32))


def tg_plan_cascade_units(plan: Plan):
    """Cascade units: (meta int32[n, 4] = KV head, first page position, end position, readers;
    readers int32[n, 256]; slots int32[n, 256]), -1 past each unit's readers."""
    n = tg_plan_get_info(plan)["n_cascade"]
    R = CASCADE_ROWS
    out = np.empty((max(n, 1), 4 + 2 * R), dtype=np.int32)
    _check(_lib().tg_plan_cascade_units(plan.handle, _hp(out)), "tg_plan_cascade_units")
    out = out[:n]
    return out[:, :4], out[:, 4:4 + R], out[:, 4 + R:]


def tg_plan_destroy(plan: Plan):
    plan.destroy()


def tg_plan_get_info(plan: Plan) -> dict:
    info = tg_plan_info()
    _check(_lib().tg_plan_get_info(plan.handle, ctypes.byref(info)), "tg_plan_get_info")
    return {f: getattr(info, f) for f, _ in tg_plan_info._fields_}


def tg_plan_items(plan: Plan) -> np.ndarray:
    """int32[n_items, 8]: bh, page_begin, page_end, tier_tokens, slot, int8 tier, worker (-1 =
    dynamic), merge index (-1 for items that write the final output)."""
    n = tg_plan_get_info(plan)["n_items"]
    out = np.empty((max(n, 1), 8), dtype=np.int32)
    _check(_lib().tg_plan_items(plan.handle, _hp(out)), "tg_plan_items")
    return out[:n]


def tg_plan_status(plan: Plan, stream=None) -> int:
    """Read and clear the device error word (synchronises the stream); returns the status."""
    return int(_lib().tg_plan_status(plan.handle, _stream(stream)))


def tg_plan_timing_enable(plan: Plan, max_calls: int):
    _check(_lib().tg_plan_timing_enable(plan.handle, max_calls), "tg_plan_timing_enable")


def tg_plan_timing_read(plan: Plan):
    """(n_calls, decode_ms_total, merge_ms_total) of the calls recorded since enable/read."""
    n = ctypes.c_int32()
    d = ctypes.c_double()
    m = ctypes.c_double()
    _check(_lib().tg_plan_timing_read(plan.handle, ctypes.byref(n), ctypes.byref(d),
                                      ctypes.byref(m)), "tg_plan_timing_read")
    return n.value, d.value, m.value


def tg_plan_trace_enable(plan: Plan, on: bool = True):
    _check(_lib().tg_plan_trace_enable(plan.handle, int(on)), "tg_plan_trace_enable")


def tg_plan_trace_read(plan: Plan, stream=None) -> np.ndarray:
    """uint64[n_workers, 8] of the last call: global-timer stamps (ns) of CTA start, first copy
    issued, first page ready, stop marker seen, worker done; dynamic items taken, split heads
    merged, ns spent merging."""
    n = tg_plan_get_info(plan)["n_workers"]
    out = np.zeros((max(n, 1), 8), dtype=np.uint64)
    _check(_lib().tg_plan_trace_read(plan.handle, _hp(out), _stream(stream)), "tg_plan_trace_read")
    return out[:n]


# ------------------------------------------------------------------------------------------
# Device entry points
# ------------------------------------------------------------------------------------------

def tg_ragged_paged_decode(plan: Plan, q, k_pages, v_pages, page_table, head_page_off,
                           head_kv_len, group_of_head, scale: float, out, lse, stream=None):
    _check_io(plan, q, out, lse)
    _check(_lib().tg_ragged_paged_decode(
        plan.handle, _dp(q), _dp(k_pages), _dp(v_pages), _dp(page_table), _dp(head_page_off),
        _dp(head_kv_len), _dp(group_of_head), float(scale), _dp(out), _dp(lse),
        _stream(stream)), "tg_ragged_paged_decode")


def tg_ragged_paged_decode_noalloc(plan: Plan, q, k_pages, v_pages, page_table, head_page_off,
                                   head_kv_len, group_of_head, scale: float, out, lse,
                                   stream=None):
    """As tg_ragged_paged_decode, for callers that cannot allocate device memory: the plan may
    be host-only; the scratch is the library's fixed 16 MiB device array."""
    _check_io(plan, q, out, lse)
    _check(_lib().tg_ragged_paged_decode_noalloc(
        plan.handle, _dp(q), _dp(k_pages), _dp(v_pages), _dp(page_table), _dp(head_page_off),
        _dp(head_kv_len), _dp(group_of_head), float(scale), _dp(out), _dp(lse),
        _stream(stream)), "tg_ragged_paged_decode_noalloc")


def tg_ragged_paged_decode_noalloc_status(stream=None) -> int:
    """Read and clear the no-alloc entry's error word on the current device (after the work
    queued on stream): TG_OK, TG_EBADPAGE or TG_ETIMEOUT."""
    return int(_lib().tg_ragged_paged_decode_noalloc_status(_stream(stream)))


def tg_ragged_paged_decode_scores(plan: Plan, q, k_pages, v_pages, page_table, head_page_off,
                                  head_kv_len, group_of_head, scale: float, out, lse,
                                  token_scores, stream=None):
    """As tg_ragged_paged_decode, also writing every retained token's scores
    s = scale * q . K_t to token_scores (fp32 [table_len * 16, G])."""
    _check_io(plan, q, out, lse)
    _check(_lib().tg_ragged_paged_decode_scores(
        plan.handle, _dp(q), _dp(k_pages), _dp(v_pages), _dp(page_table), _dp(head_page_off),
        _dp(head_kv_len), _dp(group_of_head), float(scale), _dp(out), _dp(lse),
        _dp(token_scores), _stream(stream)), "tg_ragged_paged_decode_scores")


def tg_append_sink_recent(shape: tg_shape, sink: int, k_new, v_new, k_pages, v_pages,
                          page_table, head_page_off, head_budget, head_kv_len, head_cursor,
                          slot_out, stream=None):
    """Decode-step append under the sink + recent rule (see include/tg.h)."""
    _check(_lib().tg_append_sink_recent(
        ctypes.byref(shape), int(sink), _dp(k_new), _dp(v_new), _dp(k_pages), _dp(v_pages),
        _dp(page_table), _dp(head_page_off), _dp(head_budget), _dp(head_kv_len),
        _dp(head_cursor), _dp(slot_out), _stream(stream)), "tg_append_sink_recent")


def tg_append_h2o(shape: tg_shape, k_new, v_new, k_pages, v_pages, page_table, head_page_off,
                  head_budget, head_kv_len, head_victim, slot_pos, slot_score, new_pos,
                  slot_out, stream=None):
    """Decode-step append under the H2O rule, into the slots tg_h2o_update chose."""
    _check(_lib().tg_append_h2o(
        ctypes.byref(shape), _dp(k_new), _dp(v_new), _dp(k_pages), _dp(v_pages),
        _dp(page_table), _dp(head_page_off), _dp(head_budget), _dp(head_kv_len),
        _dp(head_victim), _dp(slot_pos), _dp(slot_score), _dp(new_pos), _dp(slot_out),
        _stream(stream)), "tg_append_h2o")


def tg_h2o_update(shape: tg_shape, recent: int, token_scores, lse, head_page_off, head_budget,
                  head_kv_len, slot_pos, slot_score, next_pos, head_victim, stream=None):
    """H2O score accumulation (token_scores may be None) and the next step's victims."""
    _check(_lib().tg_h2o_update(
        ctypes.byref(shape), int(recent), _dp(token_scores), _dp(lse), _dp(head_page_off),
        _dp(head_budget), _dp(head_kv_len), _dp(slot_pos), _dp(slot_score), _dp(next_pos),
        _dp(head_victim), _stream(stream)), "tg_h2o_update")


def tg_tiered_append(shape: tg_shape, k_new, v_new, k_fast, v_fast, fast_page_table,
                     fast_head_off, head_fast_cap, k_q8, v_q8, k_scale, v_scale, slow_page_table,
                     slow_head_off, head_slow_cap, head_kv_len, head_fast_len, moved_out,
                     slot_out, stream=None):
    """Append one token per (sequence, KV head) to the fast tier, migrating the oldest fast
    token of a full window into the INT8 tier (see include/tg.h)."""
    _check(_lib().tg_tiered_append(
        ctypes.byref(shape), _dp(k_new), _dp(v_new), _dp(k_fast), _dp(v_fast),
        _dp(fast_page_table), _dp(fast_head_off), _dp(head_fast_cap), _dp(k_q8), _dp(v_q8),
        _dp(k_scale), _dp(v_scale), _dp(slow_page_table), _dp(slow_head_off),
        _dp(head_slow_cap), _dp(head_kv_len), _dp(head_fast_len), _dp(moved_out),
        _dp(slot_out), _stream(stream)), "tg_tiered_append")


def tg_tiered_append_int4(shape: tg_shape, k_new, v_new, k_fast, v_fast, fast_page_table,
                          fast_head_off, head_fast_cap, k_q4, v_q4, k_scale, v_scale,
                          slow_page_table, slow_head_off, head_slow_cap, head_kv_len,
                          head_fast_len, moved_out, slot_out, stream=None):
    """tg_tiered_append into packed INT4 pools (see include/tg.h)."""
    _check(_lib().tg_tiered_append_int4(
        ctypes.byref(shape), _dp(k_new), _dp(v_new), _dp(k_fast), _dp(v_fast),
        _dp(fast_page_table), _dp(fast_head_off), _dp(head_fast_cap), _dp(k_q4), _dp(v_q4),
        _dp(k_scale), _dp(v_scale), _dp(slow_page_table), _dp(slow_head_off),
        _dp(head_slow_cap), _dp(head_kv_len), _dp(head_fast_len), _dp(moved_out),
        _dp(slot_out), _stream(stream)), "tg_tiered_append_int4")


def tg_tiered_decode(plan: Plan, q, k_q8, v_q8, k_scale, v_scale, slow_page_table,
                     slow_head_off, k_fast, v_fast, fast_page_table, fast_head_off, head_kv_len,
                     head_fast_len, scale: float, out, lse, stream=None):
    _check_io(plan, q, out, lse)
    _check(_lib().tg_tiered_decode(
        plan.handle, _dp(q), _dp(k_q8), _dp(v_q8), _dp(k_scale), _dp(v_scale),
        _dp(slow_page_table), _dp(slow_head_off), _dp(k_fast), _dp(v_fast),
        _dp(fast_page_table), _dp(fast_head_off), _dp(head_kv_len), _dp(head_fast_len),
        float(scale), _dp(out), _dp(lse), _stream(stream)), "tg_tiered_decode")


# ------------------------------------------------------------------------------------------
# Host-buffer decode pipeline
# ------------------------------------------------------------------------------------------

def _hostp(t):
    """Host pointer of a page-locked CPU tensor."""
    if t is None or getattr(t, "is_cuda", True):
        raise ValueError("expected a CPU tensor for a host argument")
    if not t.is_pinned():
        raise ValueError("host buffers of the pipe must be page-locked (pin_memory())")
    if not t.is_contiguous():
        raise ValueError("host buffers must be contiguous")
    return t.data_ptr()


class HostPipe:
    """Owns a tg_host_pipe handle (two device staging sets, two copy streams). The host tensors
    of every call are kept alive here until wait() or destroy(), since the pipe's copies read
    and write them after the call returns."""

    def __init__(self, plan: Plan):
        h = ctypes.c_void_p()
        self._held = {}
        _check(_lib().tg_host_pipe_create(plan.handle, ctypes.byref(h)), "tg_host_pipe_create")
        self.handle = h

    def _hold(self, *tensors):
        for t in tensors:
            self._held[id(t)] = t

    def wait(self):
        _check(_lib().tg_host_pipe_wait(self.handle), "tg_host_pipe_wait")
        self._held.clear()

    def after(self, stream=None):
        _check(_lib().tg_host_pipe_after(self.handle, _stream(stream)), "tg_host_pipe_after")

    def join(self, stream=None):
        _check(_lib().tg_host_pipe_join(self.handle, _stream(stream)), "tg_host_pipe_join")

    def destroy(self):
        if self.handle:
            _lib().tg_host_pipe_destroy(self.handle)   # waits for the pipe's copies
            self.handle = ctypes.c_void_p()
        self._held.clear()

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def tg_host_pipe_create(plan: Plan) -> HostPipe:
    return HostPipe(plan)


def tg_ragged_paged_decode_host(pipe: HostPipe, plan: Plan, q_host, k_pages, v_pages, page_table,
                                head_page_off, head_kv_len, group_of_head, scale: float,
                                out_host, lse_host, stream=None):
    """tg_ragged_paged_decode with q read from, and out / lse written to, pinned host tensors
    (asynchronous: read the outputs after pipe.wait())."""
    pipe._hold(q_host, out_host, lse_host)
    _check(_lib().tg_ragged_paged_decode_host(
        pipe.handle, plan.handle, _hostp(q_host), _dp(k_pages), _dp(v_pages), _dp(page_table),
        _dp(head_page_off), _dp(head_kv_len), _dp(group_of_head), float(scale),
        _hostp(out_host), _hostp(lse_host), _stream(stream)), "tg_ragged_paged_decode_host")


def tg_tiered_decode_host(pipe: HostPipe, plan: Plan, q_host, k_q8, v_q8, k_scale, v_scale,
                          slow_page_table, slow_head_off, k_fast, v_fast, fast_page_table,
                          fast_head_off, head_kv_len, head_fast_len, scale: float, out_host,
                          lse_host, stream=None):
    """tg_tiered_decode with pinned host q / out / lse (see tg_ragged_paged_decode_host)."""
    pipe._hold(q_host, out_host, lse_host)
    _check(_lib().tg_tiered_decode_host(
        pipe.handle, plan.handle, _hostp(q_host), _dp(k_q8), _dp(v_q8), _dp(k_scale),
        _dp(v_scale), _dp(slow_page_table), _dp(slow_head_off), _dp(k_fast), _dp(v_fast),
        _dp(fast_page_table), _dp(fast_head_off), _dp(head_kv_len), _dp(head_fast_len),
        float(scale), _hostp(out_host), _hostp(lse_host), _stream(stream)),
        "tg_tiered_decode_host")


# ------------------------------------------------------------------------------------------
# TTKV slow tier in host memory, streamed block-wise
# ------------------------------------------------------------------------------------------

class SlowStream:
    """Owns a tg_slow_stream handle (per-block plans, HBM ring, copy stream). The host pools
    of its calls are kept alive here until destroy(), since the copy stream reads them after
    a call returns."""

    def __init__(self, shape: tg_shape, kv_len, fast_len, group_of_head, group_off,
                 slow_page_table, slow_head_off, block_pages: int, ring_blocks: int = 3,
                 num_workers: int = 0, min_splits: int = 1, max_chunk_pages: int = 0,
                 host_only: bool = False, device: int = -1, static_permille: int = 0,
                 dyn_chunk_pages: int = 0, early_prologue: bool = False, slow_bits: int = 8):
        self.shape = shape
        self._held = {}
        kv = _h(kv_len, np.int32).reshape(-1)
        fl = _h(fast_len, np.int32).reshape(-1)
        goh = _h(group_of_head, np.int32).reshape(-1)
        goff = _h(group_off, np.int64).reshape(-1)
        tbl = _h(slow_page_table, np.int32).reshape(-1)
        off = _h(slow_head_off, np.int64).reshape(-1)
        BH = shape.B * shape.Hkv
        _count(kv, BH, "kv_len")
        _count(fl, BH, "fast_len")
        _count(goh, shape.Hkv, "group_of_head")
        _count(goff, 2, "group_off", at_least=True)
        _count(off, BH, "slow_head_off")
        opts = tg_plan_opts(num_workers, min_splits, max_chunk_pages, int(host_only), device,
                            static_permille, dyn_chunk_pages, int(early_prologue), 0, 0, 0, 0,
                            int(slow_bits))
        h = ctypes.c_void_p()
        _check(_lib().tg_slow_stream_create(ctypes.byref(shape), _hp(kv), _hp(fl), _hp(goh),
                                            _hp(goff), goff.size - 1, _hp(tbl) if tbl.size else None,
                                            _hp(off), tbl.size, int(block_pages), int(ring_blocks),
                                            ctypes.byref(opts), ctypes.byref(h)),
               "tg_slow_stream_create")
        self.handle = h

    def blocks(self):
        """(first_page int64 [J], pages int32 [J], tokens int32 [J][B*Hkv])."""
        J = _lib().tg_slow_stream_blocks(self.handle, None, None, None)
        BH = self.shape.B * self.shape.Hkv
        first = np.empty(J, np.int64)
        pages = np.empty(J, np.int32)
        tokens = np.empty((J, BH), np.int32)
        _lib().tg_slow_stream_blocks(self.handle, _hp(first), _hp(pages), _hp(tokens))
        return first, pages, tokens

    def status(self, stream=None) -> int:
        return _lib().tg_slow_stream_status(self.handle, _stream(stream))

    def destroy(self):
        if self.handle:
            _lib().tg_slow_stream_destroy(self.handle)   # waits for the stream's copies
            self.handle = ctypes.c_void_p()
        self._held.clear()

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def tg_tiered_decode_streamed(ss: SlowStream, q, k_q8_host, v_q8_host, k_scale_host,
                              v_scale_host, k_fast, v_fast, fast_page_table, fast_head_off,
                              group_of_head, scale: float, out, lse, stream=None):
    """Tiered decode with the INT8 tier in pinned host memory, streamed block-wise."""
    rows = ss.shape.B * ss.shape.Hq
    if rows > 0:
        _bytes(q, 2 * rows * ss.shape.D, "q")
        _bytes(out, 2 * rows * ss.shape.D, "out")
        _bytes(lse, 4 * rows, "lse")
    for t in (k_q8_host, v_q8_host, k_scale_host, v_scale_host):
        ss._held[id(t)] = t
    _check(_lib().tg_tiered_decode_streamed(
        ss.handle, _dp(q), _hostp(k_q8_host), _hostp(v_q8_host), _hostp(k_scale_host),
        _hostp(v_scale_host), _dp(k_fast), _dp(v_fast), _dp(fast_page_table), _dp(fast_head_off),
        _dp(group_of_head), float(scale), _dp(out), _dp(lse), _stream(stream)),
        "tg_tiered_decode_streamed")


def tg_lse_merge(row_split_off, part_o, part_lse, out, lse, stream=None):
    n_rows = row_split_off.numel() - 1
    D = part_o.shape[-1]
    if n_rows > 0:
        _bytes(out, 2 * n_rows * D, "out")
        _bytes(lse, 4 * n_rows, "lse")
    _check(_lib().tg_lse_merge(n_rows, D, _dp(row_split_off), _dp(part_o), _dp(part_lse),
                               _dp(out), _dp(lse), _stream(stream)), "tg_lse_merge")


def tg_quantize_int8(src, codes, scale, stream=None):
    D = src.shape[-1]
    n_rows = src.numel() // D
    if n_rows > 0:
        _bytes(codes, n_rows * D, "codes")
        _bytes(scale, 4 * n_rows, "scale")
    _check(_lib().tg_quantize_int8(n_rows, D, _dp(src), _dp(codes), _dp(scale), _stream(stream)),
           "tg_quantize_int8")


def tg_quantize_int4(src, packed, scale, stream=None):
    D = src.shape[-1]
    n_rows = src.numel() // D
    if n_rows > 0:
        _bytes(packed, n_rows * D // 2, "packed")
        _bytes(scale, 4 * n_rows, "scale")
    _check(_lib().tg_quantize_int4(n_rows, D, _dp(src), _dp(packed), _dp(scale), _stream(stream)),
           "tg_quantize_int4")


# ---------------------------------------------------------------------------------------
# SplitZip codec (see include/tg.h).
# ---------------------------------------------------------------------------------------

def tg_splitzip_workspace_bytes(n: int) -> int:
    return int(_lib().tg_splitzip_workspace_bytes(int(n)))


def _bytes(t, n, what):
    """A device buffer holds at least n bytes and is contiguous (the kernels index it by n)."""
    if t is None:
        raise ValueError(f"{what}: missing")
    if t.numel() * t.element_size() < n:
        raise ValueError(f"{what}: {t.numel() * t.element_size()} bytes, {n} needed")
    if not t.is_contiguous():
        raise ValueError(f"{what}: must be contiguous")


def _zip_buffers(n, codebook, sm, codes, esc_pos, esc_exp, n_esc):
    cap = 0 if esc_pos is None else esc_pos.numel()
    _bytes(codebook, 16, "codebook")
    _bytes(n_esc, 8, "n_esc")
    if n > 0:
        _bytes(sm, n, "sm")
        _bytes(codes, (n + 1) // 2, "codes")
    if cap > 0:
        _bytes(esc_pos, 8 * cap, "esc_pos")
        _bytes(esc_exp, cap, "esc_exp")
    return cap


def tg_splitzip_encode(n: int, src, codebook, sm, codes, esc_pos, esc_exp, n_esc, workspace,
                       stream=None):
    """Encode n bf16 values of src (device); esc_cap = esc_pos.numel()."""
    n = int(n)
    cap = _zip_buffers(n, codebook, sm, codes, esc_pos, esc_exp, n_esc)
    if n > 0:
        _bytes(src, 2 * n, "src")
    _bytes(workspace, max(0, tg_splitzip_workspace_bytes(n)), "workspace")
    _check(_lib().tg_splitzip_encode(int(n), _dp(src), _dp(codebook), _dp(sm), _dp(codes),
                                     _dp(esc_pos), _dp(esc_exp), cap, _dp(n_esc),
                                     _dp(workspace), _stream(stream)), "tg_splitzip_encode")


def tg_splitzip_decode(n: int, codebook, sm, codes, esc_pos, esc_exp, n_esc, dst, stream=None):
    n = int(n)
    cap = _zip_buffers(n, codebook, sm, codes, esc_pos, esc_exp, n_esc)
    if n > 0:
        _bytes(dst, 2 * n, "dst")
    _check(_lib().tg_splitzip_decode(int(n), _dp(codebook), _dp(sm), _dp(codes), _dp(esc_pos),
                                     _dp(esc_exp), _dp(n_esc), cap, _dp(dst), _stream(stream)),
           "tg_splitzip_decode")
