"""The oracle's own derivation of a workload's layout and its fp64 reference outputs.

TEST INFRASTRUCTURE (part of the oracle): used by the tests, the smoke check and the bench's
CPU-baseline leg only. Uses synth (seeded draws) and the oracle's C functions; never the CUDA
library. The tests compare this layout with what the library derives, bit for bit, before
comparing numerics.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

import synth

import oracle


@dataclass
class OLayout:
    kv_len: np.ndarray
    fast_len: Optional[np.ndarray]
    group_of_head: np.ndarray
    n_groups: int
    num_pages: int
    page_ids: np.ndarray
    head_count: np.ndarray
    table: np.ndarray
    head_off: np.ndarray
    group_off: np.ndarray
    num_slow_pages: int = 0
    slow_ids: Optional[np.ndarray] = None
    slow_count: Optional[np.ndarray] = None
    slow_table: Optional[np.ndarray] = None
    slow_off: Optional[np.ndarray] = None


def _ceil(a, b):
    return -(-np.asarray(a, dtype=np.int64) // b)


def retained(sp, layer=0, seqs=None):
    """(kv_len int32[B, Hkv], fast_len or None); seqs selects sequences of the workload."""
    if sp.kind == "direct":
        kv, fast = synth.direct_lengths(sp, layer).astype(np.int32), None
    elif sp.kind == "ratio":
        L = np.repeat(synth.full_lengths(sp, layer)[:, None], sp.Hkv, axis=1)
        kv, fast = oracle.retained_lengths(L, synth.ratio_ppm(sp, layer)), None
    elif sp.kind == "prefix":
        _, suf = synth.prefix_layout(sp)
        kv = sp.sys_tokens + sp.doc_tokens + suf.astype(np.int64)
        kv, fast = np.repeat(kv[:, None], sp.Hkv, axis=1).astype(np.int32), None
    elif sp.kind == "tiered":
        L = np.repeat(synth.full_lengths(sp, layer)[:, None], sp.Hkv, axis=1).astype(np.int32)
        kv, fast = L, np.minimum(L, sp.fast_tokens).astype(np.int32)
    else:
        raise ValueError(sp.kind)
    if seqs is not None:
        kv = kv[seqs]
        fast = None if fast is None else fast[seqs]
    return kv, fast


def groups(sp, layer=0):
    if sp.groups == 1:
        return np.zeros(sp.Hkv, dtype=np.int32), 1
    table = synth.budget_table_ppm(sp)
    if sp.rank_over_layers:
        return oracle.budget_groups(table.reshape(-1), sp.groups).reshape(sp.layers, sp.Hkv)[layer], sp.groups
    return oracle.budget_groups(table[layer], sp.groups), sp.groups


def layout(sp, layer=0, seqs=None) -> OLayout:
    kv, fast = retained(sp, layer, seqs)
    goh, G = groups(sp, layer)
    B, H = kv.shape
    page = sp.page
    occ = lambda used: max(1, used * sp.occupancy_num // sp.occupancy_den)
    if fast is None:
        seg, chain = (), None
        if sp.kind == "prefix":
            doc, _ = synth.prefix_layout(sp)
            if seqs is not None:
                doc = doc[seqs]
            seg = [sp.sys_tokens] + [sp.doc_tokens] * sp.n_docs
            chain = np.stack([np.zeros(B, np.int32), 1 + doc], axis=1)
            shared_tok = (sp.sys_tokens // page + sp.doc_tokens // page) * page
            used = int(_ceil(kv.astype(np.int64) - shared_tok, page).sum()) + \
                sum(H * (s // page) for s in seg)
        else:
            used = int(_ceil(kv, page).sum())
        n = occ(used)
        ids, cnt, _ = oracle.reservation_layout(n, synth.free_order(sp, n, layer), page, kv, seg, chain)
        table, off, goff = oracle.group_tables(goh, G, ids, cnt)
        return OLayout(kv, None, goh, G, n, ids, cnt, table, off, goff)
    slow_n = kv - fast
    nf = occ(int(_ceil(fast, page).sum()))
    ns = occ(int(_ceil(slow_n, page).sum()))
    fids, fcnt, _ = oracle.reservation_layout(nf, synth.free_order(sp, nf, layer), page, fast)
    sids, scnt, _ = oracle.reservation_layout(ns, synth.free_order(sp, ns, layer, slow=True), page, slow_n)
    ft, foff, fgoff = oracle.group_tables(goh, G, fids, fcnt)
    st, soff, _ = oracle.group_tables(np.zeros(H, np.int32), 1, sids, scnt)
    return OLayout(kv, fast, goh, G, nf, fids, fcnt, ft, foff, fgoff, num_slow_pages=ns,
                   slow_ids=sids, slow_count=scnt, slow_table=st, slow_off=soff)


def assert_same_layout(lib_lay, o: OLayout):
    """Bit-exact equality of the library's and the oracle's layouts."""
    np.testing.assert_array_equal(lib_lay.kv_len, o.kv_len)
    if o.fast_len is not None:
        np.testing.assert_array_equal(lib_lay.fast_len, o.fast_len)
    np.testing.assert_array_equal(lib_lay.group_of_head, o.group_of_head)
    assert lib_lay.num_pages == o.num_pages
    np.testing.assert_array_equal(lib_lay.page_ids, o.page_ids)
    np.testing.assert_array_equal(lib_lay.head_count, o.head_count)
    np.testing.assert_array_equal(lib_lay.table, o.table)
    np.testing.assert_array_equal(lib_lay.head_off, o.head_off)
    np.testing.assert_array_equal(lib_lay.group_off, o.group_off)
    if o.fast_len is not None:
        assert lib_lay.num_slow_pages == o.num_slow_pages
        np.testing.assert_array_equal(lib_lay.slow_ids, o.slow_ids)
        np.testing.assert_array_equal(lib_lay.slow_table, o.slow_table)
        np.testing.assert_array_equal(lib_lay.slow_off, o.slow_off)


def q_bits(sp, layer=0, seqs=None):
    q = synth.q_bits(sp, layer)
    return q if seqs is None else np.ascontiguousarray(q[seqs])


def reference(sp, o: OLayout, layer=0, sel=None, seqs=None):
    """fp64 oracle outputs (out [rows, D], lse [rows]) of one layer; sel = rows b*Hq + hq of
    the (selected) batch."""
    q = q_bits(sp, layer, seqs)
    if o.fast_len is None:
        if sel is None:
            k = synth.pool_bits(sp, "k", o.num_pages)
            v = synth.pool_bits(sp, "v", o.num_pages)
            return oracle.decode(q, k, v, o.table, o.head_off, o.kv_len, sp.scale)
        return _sampled(sp, o, q, layer, sel)
    k = synth.pool_bits(sp, "k", o.num_pages)
    v = synth.pool_bits(sp, "v", o.num_pages)
    kq, ks, vq, vs = slow_tier(sp, o, layer)
    st = o.slow_table if o.slow_table.size else np.zeros(1, np.int32)
    return oracle.tiered_decode(q, kq, vq, ks, vs, st, o.slow_off, k, v, o.table, o.head_off,
                                o.kv_len, o.fast_len, sp.scale, sel=sel)


def slow_tier(sp, o: OLayout, layer=0):
    """The quantised slow tier as the oracle stores it: (k codes, k scales, v codes, v scales),
    codes int8 [Ps][page][D] (INT4 tiers unpacked from their packed form)."""
    kb = synth.pool_bits(sp, "kslow", o.num_slow_pages)
    vb = synth.pool_bits(sp, "vslow", o.num_slow_pages)
    if getattr(sp, "slow_bits", 8) == 4:
        kp, ks = oracle.quantize_int4(kb)
        vp, vs = oracle.quantize_int4(vb)
        return oracle.unpack_int4(kp), ks, oracle.unpack_int4(vp), vs
    kq, ks = oracle.quantize_int8(kb)
    vq, vs = oracle.quantize_int8(vb)
    return kq, ks, vq, vs


def _sampled(sp, o, q, layer, sel):
    """Oracle outputs of selected rows at full size: gather only the pages those rows read
    into a compact pool, with a remapped table (the values are those of the full pool)."""
    sel = np.asarray(sel, dtype=np.int64)
    G = sp.Hq // sp.Hkv
    bh = np.unique((sel // sp.Hq) * sp.Hkv + (sel % sp.Hq) // G)
    pages = []
    for x in bh:
        n = int(o.head_count.reshape(-1)[x])
        off = int(o.head_off.reshape(-1)[x])
        pages.append(o.table[off:off + n])
    uniq = np.unique(np.concatenate(pages))
    k = synth.pool_page_bits(sp, "k", uniq)
    v = synth.pool_page_bits(sp, "v", uniq)
    table = _remap(o.table, uniq)
    return oracle.decode(q, k, v, table, o.head_off, o.kv_len, sp.scale, sel=sel)


def _remap(table, uniq):
    pos = np.searchsorted(uniq, table)
    pos = np.clip(pos, 0, len(uniq) - 1)
    hit = (table >= 0) & (uniq[pos] == table)
    return np.where(hit, pos, -1).astype(np.int32)
