"""Admission of a synthetic decode workload through libtg's host steps.

Given a workload shape (synth.Spec) and a layer, this runs the library's admission-time steps
— retained lengths from the budget table, budget groups, Budget Reservation from a seeded free
list (shared prefix segments first), group page tables, the static plan — and uploads the
seeded pool contents and queries to the device. It is the serving-engine side of one decode
step: everything here happens once per admission, never per step.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

import synth
from . import (make_shape, tg_alloc_create, tg_alloc_destroy, tg_alloc_free_pages, tg_reserve,
               tg_share_segment, tg_budget_groups, tg_build_group_tables, tg_plan_create,
               tg_quantize_int4, tg_quantize_int8, tg_retained_lengths)


@dataclass
class Layout:
    """Host-side layout of one layer (all numpy)."""
    kv_len: np.ndarray          # int32[B, Hkv]
    fast_len: Optional[np.ndarray]
    group_of_head: np.ndarray   # int32[Hkv]
    n_groups: int
    num_pages: int
    page_ids: np.ndarray        # flat, (b, h, page) order
    head_count: np.ndarray      # int32[B, Hkv]
    table: np.ndarray
    head_off: np.ndarray        # int64[B, Hkv]
    group_off: np.ndarray       # int64[n_groups + 1]
    # tiered only: the INT8 tier's layout
    num_slow_pages: int = 0
    slow_ids: Optional[np.ndarray] = None
    slow_count: Optional[np.ndarray] = None
    slow_table: Optional[np.ndarray] = None
    slow_off: Optional[np.ndarray] = None
    seg_pages: Optional[np.ndarray] = None


def pages_of(n, page=16):
    return (np.asarray(n, dtype=np.int64) + page - 1) // page


def _occupied(sp: synth.Spec, used: int) -> int:
    return max(1, used * sp.occupancy_num // sp.occupancy_den)


def retained(sp: synth.Spec, layer: int = 0, seqs=None):
    """(kv_len int32[B, Hkv], fast_len or None) of one layer, via the library; seqs selects
    sequences of the workload (a shard)."""
    if sp.kind == "direct":
        kv, fast = synth.direct_lengths(sp, layer).astype(np.int32), None
    elif sp.kind == "ratio":
        L = np.repeat(synth.full_lengths(sp, layer)[:, None], sp.Hkv, axis=1)
        kv, fast = tg_retained_lengths(L, synth.ratio_ppm(sp, layer)), None
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
        kv = np.ascontiguousarray(kv[seqs])
        fast = None if fast is None else np.ascontiguousarray(fast[seqs])
    return kv, fast


def groups(sp: synth.Spec, layer: int = 0):
    """group_of_head int32[Hkv] of one layer and the number of groups, via the library."""
    if sp.groups == 1:
        return np.zeros(sp.Hkv, dtype=np.int32), 1
    table = synth.budget_table_ppm(sp)
    if sp.rank_over_layers:
        g = tg_budget_groups(table.reshape(-1), sp.groups).reshape(sp.layers, sp.Hkv)
        return g[layer].astype(np.int32), sp.groups
    return tg_budget_groups(table[layer], sp.groups), sp.groups


def _reserve(sp, num_pages, seed, kv, segs=(), chain=None):
    """Budget Reservation of every sequence from a pool the library shuffles with `seed`
    (shared segments first; chain[b] lists the segments sequence b extends). Returns the page
    ids flat, each head's page count int32[B, Hkv] and the shared segments' pages."""
    B, H = kv.shape
    a = tg_alloc_create(num_pages, sp.page, seed)
    try:
        seg_ids, seg_pages = [], []
        for n_tok in segs:
            sid, ids = tg_share_segment(a, int(n_tok), H, sp.page)
            seg_ids.append(sid)
            seg_pages.append(ids.reshape(-1))
        out, counts = [], np.zeros((B, H), np.int32)
        for b in range(B):
            pre = () if chain is None else [seg_ids[c] for c in chain[b]]
            ids, counts[b] = tg_reserve(a, b, kv[b], pre, sp.page, with_counts=True)
            out.append(ids)
        ids = np.concatenate(out) if out else np.zeros(0, np.int32)
        sp_all = np.concatenate(seg_pages) if seg_pages else np.zeros(0, np.int32)
        return ids.astype(np.int32), counts, sp_all.astype(np.int32)
    finally:
        tg_alloc_destroy(a)


def _pages_used(sp, kv, segs=(), chain=None) -> int:
    """Pages a reservation of these heads takes (each shared segment's pages once, then every
    head's private pages), as the allocator counts them: its free pages before minus after, in
    a pool with room for any reservation of these lengths."""
    H = kv.shape[1]
    room = int(kv.astype(np.int64).sum()) // sp.page + kv.size + H * sum(int(t) // sp.page for t in segs) + 1
    a = tg_alloc_create(room, sp.page, 0)
    try:
        before = tg_alloc_free_pages(a)
        seg_ids = [tg_share_segment(a, int(t), H, sp.page)[0] for t in segs]
        for b in range(kv.shape[0]):
            tg_reserve(a, b, kv[b], () if chain is None else [seg_ids[c] for c in chain[b]], sp.page)
        return int(before - tg_alloc_free_pages(a))
    finally:
        tg_alloc_destroy(a)


def layout(sp: synth.Spec, layer: int = 0, seqs=None) -> Layout:
    kv, fast = retained(sp, layer, seqs)
    goh, G = groups(sp, layer)
    B, H = kv.shape
    segs, chain = (), None
    if sp.kind == "prefix":
        segs = [sp.sys_tokens] + [sp.doc_tokens] * sp.n_docs
        doc, _ = synth.prefix_layout(sp)
        if seqs is not None:
            doc = doc[seqs]
        chain = np.stack([np.zeros(B, np.int32), 1 + doc], axis=1)
    if fast is None:
        # the pool is sized from the pages the workload uses (its occupancy): the reservation
        # is made once in a pool with room for every page, which gives the pages in use, then
        # in the pool of the workload's size
        used = _pages_used(sp, kv, segs, chain)
        num_pages = _occupied(sp, used)
        ids, count, segp = _reserve(sp, num_pages, synth.free_order_seed(sp, layer), kv, segs, chain)
        table, off, goff = tg_build_group_tables(count, goh, G, ids)
        return Layout(kv, None, goh, G, num_pages, ids, count, table, off, goff, seg_pages=segp)
    slow_n = kv - fast
    nf = _occupied(sp, _pages_used(sp, fast))
    ns = _occupied(sp, _pages_used(sp, slow_n))
    fids, fcount, _ = _reserve(sp, nf, synth.free_order_seed(sp, layer), fast)
    sids, scount, _ = _reserve(sp, ns, synth.free_order_seed(sp, layer, slow=True), slow_n)
    ft, foff, fgoff = tg_build_group_tables(fcount, goh, G, fids)
    st, soff, sgoff = tg_build_group_tables(scount, np.zeros(H, np.int32), 1, sids)
    return Layout(kv, fast, goh, G, nf, fids, fcount, ft, foff, fgoff, num_slow_pages=ns,
                  slow_ids=sids, slow_count=scount, slow_table=st, slow_off=soff)


@dataclass
class DeviceBatch:
    """Device tensors of one layer's decode step, and its plan."""
    spec: synth.Spec
    lay: Layout
    plan: object
    q: object
    out: object
    lse: object
    k: object = None
    v: object = None
    table: object = None
    head_off: object = None
    kv_len: object = None
    group_of_head: object = None
    # tiered
    k_q8: object = None
    v_q8: object = None
    k_scale: object = None
    v_scale: object = None
    slow_table: object = None
    slow_off: object = None
    fast_len: object = None
    extra: dict = field(default_factory=dict)

    def run(self, stream=None):
        from . import tg_ragged_paged_decode, tg_tiered_decode
        if self.lay.fast_len is None:
            tg_ragged_paged_decode(self.plan, self.q, self.k, self.v, self.table, self.head_off,
                                   self.kv_len, self.group_of_head, self.spec.scale, self.out,
                                   self.lse, stream)
        else:
            tg_tiered_decode(self.plan, self.q, self.k_q8, self.v_q8, self.k_scale, self.v_scale,
                             self.slow_table, self.slow_off, self.k, self.v, self.table,
                             self.head_off, self.kv_len, self.fast_len, self.spec.scale,
                             self.out, self.lse, stream)


    def run_host(self, pipe, q_host, out_host, lse_host, stream=None):
        """One decode step through the host-buffer pipe (pinned q in, out / lse back)."""
        from . import tg_ragged_paged_decode_host, tg_tiered_decode_host
        if self.lay.fast_len is None:
            tg_ragged_paged_decode_host(pipe, self.plan, q_host, self.k, self.v, self.table,
                                        self.head_off, self.kv_len, self.group_of_head,
                                        self.spec.scale, out_host, lse_host, stream)
        else:
            tg_tiered_decode_host(pipe, self.plan, q_host, self.k_q8, self.v_q8, self.k_scale,
                                  self.v_scale, self.slow_table, self.slow_off, self.k, self.v,
                                  self.table, self.head_off, self.kv_len, self.fast_len,
                                  self.spec.scale, out_host, lse_host, stream)


    def host_slow_tier(self):
        """Page-locked host copies of the INT8 tier: (k codes, v codes, k scales, v scales)."""
        return tuple(t.cpu().pin_memory() for t in (self.k_q8, self.v_q8, self.k_scale, self.v_scale))

    def slow_stream(self, block_pages: int, ring_blocks: int = 3, **kw):
        """A tg_slow_stream over this batch's tiers (the INT8 tier to be read from host)."""
        from . import SlowStream
        lay = self.lay
        dev = self.q.device.index
        return SlowStream(self.plan.shape, lay.kv_len, lay.fast_len, lay.group_of_head,
                          lay.group_off, lay.slow_table if lay.slow_table.size else np.full(1, -1),
                          lay.slow_off, block_pages, ring_blocks,
                          device=dev if dev is not None else -1, slow_bits=self.spec.slow_bits,
                          **kw)

    def run_streamed(self, ss, host, stream=None):
        """One tiered step with the INT8 tier streamed from the pinned host copies `host`."""
        from . import tg_tiered_decode_streamed
        tg_tiered_decode_streamed(ss, self.q, *host, self.k, self.v, self.table, self.head_off,
                                  self.group_of_head, self.spec.scale, self.out, self.lse, stream)


def timed_plan_options(cfg: int) -> dict:
    """Plan options per workload, chosen by measurement on B200, the ones bench.py times: the
    static share of the bytes, the largest dynamic item, the cascade for shared prefixes, and
    early prologue (only this library's kernels run back to back, so the decode may read its
    plan and tables before the previous step's merge kernel has finished)."""
    kw = dict(early_prologue=True)
    if cfg == 1:
        # one tiny batch: whole heads, so a step is one launch (no split head, no merge)
        kw.update(whole_heads=True)
    elif cfg == 2:
        kw.update(static_permille=850, dyn_chunk_pages=16)
    elif cfg == 3:
        kw.update(static_permille=900, dyn_chunk_pages=32)
    elif cfg == 4:
        # shared prefix pages: the cascade reads each shared run once per step for all its
        # readers; the private pages stay on the split-K items. The decode kernel's CTAs start
        # as the cascade's finish, so less of its work is placed ahead of time
        kw.update(static_permille=400, dyn_chunk_pages=16, cascade=True)
    elif cfg == 5:
        kw.update(min_splits=64, max_chunk_pages=128, static_permille=900, dyn_chunk_pages=32)
    return kw


def _bf16_tensor(bits: np.ndarray, device):
    import torch
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)


def _pool_to_device(sp, which, n, device, chunk_pages=1 << 16):
    """Generate a pool on the host in chunks and copy it to the device. The contents do not
    depend on the layer (see synth.pool_bits)."""
    import torch
    out = torch.empty((n, sp.page, sp.D), dtype=torch.bfloat16, device=device)
    per = sp.page * sp.D
    kind = {"k": synth.S_K, "v": synth.S_V, "kslow": synth.S_KSLOW, "vslow": synth.S_VSLOW}[which]
    buf = np.empty(min(n, chunk_pages) * per, dtype=np.uint16)
    for p0 in range(0, n, chunk_pages):
        c = min(chunk_pages, n - p0)
        synth.normal_bf16(sp.seed, synth.stream_id(kind), c * per, i0=p0 * per,
                          out=buf[:c * per])
        out[p0:p0 + c].copy_(torch.from_numpy(buf[:c * per].view(np.int16)).view(torch.bfloat16)
                             .view(c, sp.page, sp.D), non_blocking=False)
    return out


def pools_to_device(sp: synth.Spec, num_pages: int, device="cuda"):
    """The bf16 K and V pools of num_pages pages on the device. A layer whose pool has n <=
    num_pages pages reads the first n of them (the same bytes its own pool would hold), so one
    upload serves every layer of a multi-layer workload."""
    return (_pool_to_device(sp, "k", num_pages, device), _pool_to_device(sp, "v", num_pages, device))


def to_device(sp: synth.Spec, lay: Layout, layer: int = 0, device="cuda", num_workers: int = 0,
              min_splits: int = 1, max_chunk_pages: int = 0, seqs=None, static_permille: int = 0,
              dyn_chunk_pages: int = 0, early_prologue: bool = False, wait_limit_us: int = 0,
              test_withhold_page: int = 0, cascade: bool = False,
              min_readers: int = 2, whole_heads: bool = False, pools=None) -> DeviceBatch:
    """Upload one layer's tables, lengths and queries, make its plan, and upload (or, with
    pools = (k, v) from pools_to_device holding at least lay.num_pages pages, reuse) its bf16
    K and V pools."""
    import torch
    dev = torch.device(device)
    B = lay.kv_len.shape[0]
    shape = make_shape(B, sp.Hq, sp.Hkv, sp.D, lay.num_pages, lay.num_slow_pages, sp.page)
    if cascade:
        from . import tg_plan_create_cascade
        plan = tg_plan_create_cascade(
            shape, lay.kv_len, lay.group_of_head, lay.group_off,
            lay.table if lay.table.size else np.full(1, -1), lay.head_off,
            min_readers=min_readers, num_workers=num_workers, min_splits=min_splits,
            max_chunk_pages=max_chunk_pages, static_permille=static_permille,
            dyn_chunk_pages=dyn_chunk_pages, early_prologue=early_prologue,
            wait_limit_us=wait_limit_us, device=dev.index if dev.index is not None else -1)
    else:
        plan = tg_plan_create(shape, lay.kv_len, lay.group_of_head, lay.group_off,
                              fast_len=lay.fast_len,
                              slow_table_len=0 if lay.slow_table is None else lay.slow_table.size,
                              num_workers=num_workers, min_splits=min_splits,
                              max_chunk_pages=max_chunk_pages, static_permille=static_permille,
                              dyn_chunk_pages=dyn_chunk_pages, early_prologue=early_prologue,
                              wait_limit_us=wait_limit_us, test_withhold_page=test_withhold_page,
                              device=dev.index if dev.index is not None else -1,
                              slow_bits=sp.slow_bits if lay.fast_len is not None else 8,
                              whole_heads=whole_heads)
    qb = synth.q_bits(sp, layer)
    q = _bf16_tensor(qb if seqs is None else np.ascontiguousarray(qb[seqs]), dev)
    out = torch.empty((B, sp.Hq, sp.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, sp.Hq), dtype=torch.float32, device=dev)
    it = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dtype=dt)).to(dev)
    db = DeviceBatch(sp, lay, plan, q, out, lse)
    if pools is not None:
        assert pools[0].shape[0] >= lay.num_pages and pools[1].shape[0] >= lay.num_pages
        db.k, db.v = pools[0][:lay.num_pages], pools[1][:lay.num_pages]
    else:
        db.k = _pool_to_device(sp, "k", lay.num_pages, dev)
        db.v = _pool_to_device(sp, "v", lay.num_pages, dev)
    db.table = it(lay.table if lay.table.size else np.full(1, -1), np.int32)
    db.head_off = it(lay.head_off, np.int64)
    db.kv_len = it(lay.kv_len, np.int32)
    db.group_of_head = it(lay.group_of_head, np.int32)
    if lay.fast_len is not None:
        ns = lay.num_slow_pages
        db.fast_len = it(lay.fast_len, np.int32)
        db.slow_table = it(lay.slow_table if lay.slow_table.size else np.full(1, -1), np.int32)
        db.slow_off = it(lay.slow_off, np.int64)
        # INT8 pools int8 [ns][page][D]; INT4 pools packed uint8 [ns][page][D/2]
        i4 = sp.slow_bits == 4
        cshape, cdt = ((ns, sp.page, sp.D // 2), torch.uint8) if i4 else ((ns, sp.page, sp.D), torch.int8)
        db.k_q8 = torch.empty(cshape, dtype=cdt, device=dev)
        db.v_q8 = torch.empty(cshape, dtype=cdt, device=dev)
        db.k_scale = torch.empty((ns, sp.page), dtype=torch.float32, device=dev)
        db.v_scale = torch.empty((ns, sp.page), dtype=torch.float32, device=dev)
        for which, codes, scale in (("kslow", db.k_q8, db.k_scale), ("vslow", db.v_q8, db.v_scale)):
            src = _pool_to_device(sp, which, ns, dev)
            (tg_quantize_int4 if i4 else tg_quantize_int8)(src, codes, scale)
            del src
        torch.cuda.synchronize(dev)
    return db


def admit(sp: synth.Spec, layer: int = 0, device="cuda", seqs=None, **plan_kw) -> DeviceBatch:
    return to_device(sp, layout(sp, layer, seqs), layer, device, seqs=seqs, **plan_kw)


def algorithmic_bytes(sp: synth.Spec, lay: Layout) -> dict:
    """Bytes one decode step must move: retained K/V (INT8 / INT4 scales included), the page-table
    entries and per-head table words read, q in, out + lse written."""
    kv = lay.kv_len.astype(np.int64)
    if lay.fast_len is None:
        kvb = int(kv.sum()) * 2 * sp.D * 2
        tab = int(pages_of(kv, sp.page).sum()) * 4
    else:
        f = np.minimum(lay.fast_len.astype(np.int64), kv)
        row = sp.D // 2 if sp.slow_bits == 4 else sp.D   # code bytes per slow token and tensor
        kvb = int((kv - f).sum()) * 2 * (row + 4) + int(f.sum()) * 2 * sp.D * 2
        tab = int((pages_of(kv - f, sp.page) + pages_of(f, sp.page)).sum()) * 4
    B = lay.kv_len.shape[0]
    BH = B * sp.Hkv
    heads = BH * (8 + 4 + (8 + 4 if lay.fast_len is not None else 0))  # offsets + lengths
    qo = B * sp.Hq * sp.D * 2 * 2 + B * sp.Hq * 4
    return {"kv": kvb, "tables": tab + heads, "q_out": qo, "total": kvb + tab + heads + qo}
