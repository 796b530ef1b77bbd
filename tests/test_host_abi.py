"""CPU tests of the C ABI: the library loads and exports every declared symbol, and its host
steps (retained lengths, groups, reservation, group tables, placement, the planner) agree bit
for bit with the oracle's own derivation. No device calls."""
import ctypes
import os
import re

import numpy as np
import pytest

import non_uniform_paged_flash_b200 as tg
import oracle
import synth
from non_uniform_paged_flash_b200 import workload
from tests import _oracle_side as ors

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_library_exports_every_declared_symbol():
    hdr = open(os.path.join(ROOT, "include", "tg.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    declared = set(re.findall(r"\b(tg_[a-z0-9_]+)\s*\(", hdr))
    assert declared, "no declarations parsed"
    lib = tg.load()
    for name in sorted(declared):
        assert hasattr(lib, name), f"libtg.so does not export {name}"
    assert declared == set(tg.ABI_SYMBOLS), declared ^ set(tg.ABI_SYMBOLS)


# The calls the hot path's boundary names (the scope table's C-ABI sketch), by name.
BOUNDARY_CALLS = ("tg_alloc_create", "tg_reserve", "tg_share_segment", "tg_release",
                  "tg_alloc_destroy", "tg_build_group_tables", "tg_plan_create",
                  "tg_ragged_paged_decode", "tg_tiered_decode", "tg_plan_destroy", "tg_strerror")


def test_boundary_calls_are_exported_under_their_names():
    hdr = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "tg.h")).read(), flags=re.S)
    lib = tg.load()
    for name in BOUNDARY_CALLS:
        assert re.search(r"\b%s\s*\(" % name, hdr), f"tg.h does not declare {name}"
        assert hasattr(lib, name), f"libtg.so does not export {name}"
    # and the host ones run through the C ABI here (the device ones need a GPU)
    a = tg.tg_alloc_create(64, 16, 9)
    sid, _ = tg.tg_share_segment(a, 32, 2, 16)
    ids, counts = tg.tg_reserve(a, 0, [40, 33], (sid,), 16, with_counts=True)
    table, off, goff = tg.tg_build_group_tables(counts.reshape(1, 2), [0, 0], 1, ids)
    assert table.tolist() == ids.tolist() and counts.tolist() == [3, 3]
    tg.tg_release(a, 0)
    tg.tg_alloc_destroy(a)
    assert tg.load().tg_strerror(0).decode() == "ok"


def test_strerror_covers_codes():
    for code in range(10):
        assert tg.load().tg_strerror(code).decode() != "unknown status"


def test_retained_lengths_match_oracle():
    rng = np.random.default_rng(20)
    L = rng.integers(-3, 300_000, 20_000).astype(np.int32)
    r = rng.integers(0, 1_000_001, 20_000).astype(np.int32)
    np.testing.assert_array_equal(tg.tg_retained_lengths(L, r), oracle.retained_lengths(L, r))
    with pytest.raises(tg.TGError):
        tg.tg_retained_lengths([10], [1_000_001])


def test_budget_groups_match_oracle():
    rng = np.random.default_rng(21)
    for n, G in [(8, 4), (256, 8), (13, 5), (8, 8), (1, 1)]:
        b = rng.integers(0, 50, n).astype(np.int32)   # many ties
        np.testing.assert_array_equal(tg.tg_budget_groups(b, G), oracle.budget_groups(b, G))
    with pytest.raises(tg.TGError):
        tg.tg_budget_groups([1, 2], 3)


def _lib_reservation(num_pages, order, kv, segs=(), chain=None, page=16):
    a = tg.tg_alloc_create_ordered(num_pages, page, order)
    try:
        seg_ids = []
        seg_pages = []
        for s in segs:
            sid, ids = tg.tg_share_segment(a, s, kv.shape[1], page)
            seg_ids.append(sid)
            seg_pages.append(ids.reshape(-1))
        out = []
        for b in range(kv.shape[0]):
            pre = [] if chain is None else [seg_ids[c] if c >= 0 else -1 for c in chain[b]]
            out.append(tg.tg_reserve(a, b, kv[b], pre, page))
        return np.concatenate(out), (np.concatenate(seg_pages) if seg_pages else np.zeros(0, np.int32))
    finally:
        tg.tg_alloc_destroy(a)


def test_reservation_matches_oracle_plain_and_prefix():
    rng = np.random.default_rng(22)
    kv = rng.integers(0, 400, (11, 3)).astype(np.int32)
    need = int(((kv + 15) // 16).sum())
    order = rng.permutation(need + 5).astype(np.int32)
    ids, _ = _lib_reservation(need + 5, order, kv)
    oids, _, _ = oracle.reservation_layout(need + 5, order, 16, kv)
    np.testing.assert_array_equal(ids, oids)
    # prefix sharing with partial segments and an absent chain entry
    segs = [100, 37, 64]
    chain = np.array([[0, 1], [0, 2], [0, -1], [-1, 2], [0, 1]])
    shared = np.array([sum(segs[c] // 16 * 16 for c in row if c >= 0) for row in chain])
    kv = (shared[:, None] + rng.integers(0, 70, (5, 2))).astype(np.int32)
    order = rng.permutation(400).astype(np.int32)
    ids, segp = _lib_reservation(400, order, kv, segs, chain)
    oids, _, osegp = oracle.reservation_layout(400, order, 16, kv, segs, chain)
    np.testing.assert_array_equal(ids, oids)
    np.testing.assert_array_equal(segp, osegp)


def test_reservation_is_all_or_nothing():
    a = tg.tg_alloc_create_ordered(10, 16, np.arange(10)[::-1])
    try:
        tg.tg_reserve(a, 0, [40, 16])                       # 3 + 1 pages
        assert tg.tg_alloc_free_pages(a) == 6
        with pytest.raises(tg.TGError) as e:
            tg.tg_reserve(a, 1, [64, 64])                   # needs 8 > 6
        assert e.value.status == tg.TG_ENOSPC
        assert tg.tg_alloc_free_pages(a) == 6                     # unchanged
        ids = tg.tg_reserve(a, 1, [32, 1])                  # same as if no failure
        np.testing.assert_array_equal(ids, [5, 4, 3])
        with pytest.raises(tg.TGError) as e:
            tg.tg_reserve(a, 1, [1])
        assert e.value.status == tg.TG_EEXIST
        with pytest.raises(tg.TGError) as e:
            tg.tg_release(a, 7)
        assert e.value.status == tg.TG_ENOTFOUND
    finally:
        tg.tg_alloc_destroy(a)


def test_free_order_must_be_a_permutation():
    with pytest.raises(tg.TGError):
        tg.tg_alloc_create_ordered(4, 16, [0, 1, 1, 2])
    with pytest.raises(tg.TGError):
        tg.tg_alloc_create_ordered(3, 16, [0, 1, 3])


def test_shared_segment_refcounts_and_release_order():
    a = tg.tg_alloc_create_ordered(40, 16)
    try:
        sid, sp = tg.tg_share_segment(a, 40, 2, 16)         # 2 full pages per head
        np.testing.assert_array_equal(sp, [[0, 1], [2, 3]])
        r0 = tg.tg_reserve(a, 0, [50, 33], [sid])          # shared 32 tokens
        r1 = tg.tg_reserve(a, 1, [32, 40], [sid])
        np.testing.assert_array_equal(r0, [0, 1, 4, 5, 2, 3, 6])
        np.testing.assert_array_equal(r1, [0, 1, 2, 3, 7])
        for p in (0, 1, 2, 3):
            assert tg.tg_alloc_refcount(a, p) == 3                # segment + 2 readers
        assert tg.tg_alloc_refcount(a, 4) == 1
        tg.tg_release(a, 0)
        assert tg.tg_alloc_refcount(a, 0) == 2 and tg.tg_alloc_refcount(a, 4) == 0
        free_before = tg.tg_alloc_free_pages(a)
        tg.tg_release_segment(a, sid)
        assert tg.tg_alloc_free_pages(a) == free_before           # reader 1 still holds them
        tg.tg_release(a, 1)
        assert all(tg.tg_alloc_refcount(a, p) == 0 for p in range(8))
        assert tg.tg_alloc_free_pages(a) == 40
        # released pages are appended at the back, in release order: the front is unchanged
        ids = tg.tg_reserve(a, 2, [16])
        np.testing.assert_array_equal(ids, [8])
        with pytest.raises(tg.TGError):
            tg.tg_reserve(a, 3, [16], [sid])               # dead segment
    finally:
        tg.tg_alloc_destroy(a)


def test_group_tables_match_oracle():
    rng = np.random.default_rng(23)
    for B, H, G in [(7, 8, 4), (3, 5, 5), (4, 4, 1), (6, 8, 8)]:
        cnt = rng.integers(0, 9, (B, H)).astype(np.int32)
        goh = rng.integers(0, G, H).astype(np.int32)
        ids = rng.permutation(int(cnt.sum()) + 3)[: int(cnt.sum())].astype(np.int32)
        t, off, goff = tg.tg_build_group_tables(cnt, goh, G, ids)
        ot, ooff, ogoff = oracle.group_tables(goh, G, ids, cnt)
        np.testing.assert_array_equal(t, ot)
        np.testing.assert_array_equal(goff, ogoff)
        # head_off of empty groups' heads is only meaningful where the head has pages
        np.testing.assert_array_equal(off, ooff)


def test_place_sequences_match_oracle():
    rng = np.random.default_rng(24)
    for n, g in [(64, 2), (513, 8), (5, 7), (1000, 3)]:
        b = rng.integers(0, 10**7, n)
        b[::7] = b[0]                                              # ties
        np.testing.assert_array_equal(tg.tg_place_sequences(b, g), oracle.place_sequences(b, g))


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_small_workload_layout_matches_oracle(cfg):
    sp = synth.small(cfg)
    for layer in range(min(sp.layers, 3)):
        ors.assert_same_layout(workload.layout(sp, layer), ors.layout(sp, layer))


@pytest.mark.parametrize("cfg", [2, 4, 5])
def test_full_size_layout_matches_oracle(cfg):
    sp = synth.preset(cfg)
    ors.assert_same_layout(workload.layout(sp, 0), ors.layout(sp, 0))


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_pool_occupancy_as_specified(cfg):
    """Pool sizes against the workloads' own statement, not against the shared formula: the tiny
    workload's pool is exactly the used pages; the GQA layer's and the serving step's pools are
    floor(used * 10 / 9) pages, so at least 90 % occupied, and one page more would not be."""
    sp = synth.preset(cfg)
    lay = workload.layout(sp, 0)
    used = int(lay.head_count.sum())
    assert used == int(((lay.kv_len.astype(np.int64) + 15) // 16).sum())
    if cfg == 1:
        assert lay.num_pages == used
    else:
        assert lay.num_pages == used * 10 // 9
        assert used / lay.num_pages >= 0.9
        assert used / (lay.num_pages + 1) < 0.9
    ids = np.asarray(lay.page_ids)
    assert len(np.unique(ids)) == used and ids.min() >= 0 and ids.max() < lay.num_pages


def test_full_size_layout_matches_oracle_multi_layer():
    sp = synth.preset(3)
    for layer in (0, 31):
        ors.assert_same_layout(workload.layout(sp, layer), ors.layout(sp, layer))


# ---------------------------------------------------------------------------------------
# Planner (host-only plans)
# ---------------------------------------------------------------------------------------

def test_hybrid_plan_static_share():
    """With static_permille = 800 every worker's static bytes are ~80% of its fair share."""
    sp = synth.preset(2)
    lay = workload.layout(sp, 0)
    W = 592
    p = _plan(sp, lay, num_workers=W, static_permille=800)
    items = tg.tg_plan_items(p)
    _check_coverage(sp, lay, items)
    _check_merge_indices(items)
    st = items[:, 6] >= 0
    pages = (items[:, 2] - items[:, 1]).astype(np.int64)
    per_w = np.bincount(items[st, 6], weights=pages[st], minlength=W)
    total = pages.sum()
    assert abs(per_w.mean() - 0.8 * total / W) <= 2
    assert per_w.max() - per_w.min() <= 4
    assert abs(pages[~st].sum() - 0.2 * total) <= 0.01 * total


def _plan(sp, lay, **kw):
    shape = tg.make_shape(sp.B, sp.Hq, sp.Hkv, sp.D, lay.num_pages, lay.num_slow_pages, sp.page)
    return tg.tg_plan_create(shape, lay.kv_len, lay.group_of_head, lay.group_off,
                             fast_len=lay.fast_len,
                             slow_table_len=0 if lay.slow_table is None else lay.slow_table.size,
                             host_only=True, **kw)


def _check_coverage(sp, lay, items, min_splits=1, max_chunk=0):
    """Every (head, tier, page) is covered exactly once; items stay in one tier; slots of a
    split head are consecutive in item order; single-item heads write the final output."""
    kv = lay.kv_len.reshape(-1).astype(np.int64)
    fl = None if lay.fast_len is None else lay.fast_len.reshape(-1).astype(np.int64)
    seen = {}
    for bh, pb, pe, tier_tok, slot, flags, worker, _ in items:
        assert 0 <= pb < pe
        slow = bool(flags & 1)
        n = kv[bh] if fl is None else (kv[bh] - min(fl[bh], kv[bh]) if slow else min(fl[bh], kv[bh]))
        assert tier_tok == n
        assert pe <= -(-n // 16)
        if max_chunk:
            assert pe - pb <= max_chunk
        for p in range(pb, pe):
            key = (bh, slow, p)
            assert key not in seen, key
            seen[key] = slot
    want = 0
    for bh in range(kv.size):
        if fl is None:
            want += -(-kv[bh] // 16)
        else:
            f = min(fl[bh], kv[bh])
            want += -(-(kv[bh] - f) // 16) + -(-f // 16)
    assert len(seen) == want
    by_head = {}
    for row in items:
        by_head.setdefault(int(row[0]), []).append(int(row[4]))
    for bh, slots in by_head.items():
        if len(slots) == 1:
            assert slots == [-1]
        else:
            assert slots == list(range(slots[0], slots[0] + len(slots)))
            if min_splits > 1:
                assert len(slots) >= min(min_splits, sum(1 for r in items if r[0] == bh))


def _check_merge_indices(items):
    """Split heads: one merge index per head, distinct across heads; final items have none."""
    by_head = {}
    for bh, pb, pe, tt, slot, tier, worker, mi in items:
        if slot < 0:
            assert mi == -1
        else:
            assert mi >= 0
            by_head.setdefault(int(bh), set()).add(int(mi))
    idx = [next(iter(v)) for v in by_head.values()]
    assert all(len(v) == 1 for v in by_head.values())
    assert sorted(idx) == list(range(len(idx)))


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("workers", [1, 7, 592])
@pytest.mark.parametrize("static_permille", [1000, 800, 300])
def test_plan_coverage(cfg, workers, static_permille):
    sp = synth.small(cfg)
    lay = workload.layout(sp, 0)
    p = _plan(sp, lay, num_workers=workers, static_permille=static_permille)
    items = tg.tg_plan_items(p)
    _check_coverage(sp, lay, items)
    _check_merge_indices(items)
    info = tg.tg_plan_get_info(p)
    assert info["n_items"] == len(items) and info["n_workers"] <= workers
    assert info["n_empty"] == int((lay.kv_len == 0).sum())
    dyn = items[:, 6] == -1
    assert info["n_dynamic"] == int(dyn.sum())
    if static_permille == 1000:
        assert not dyn.any()
    if dyn.any():
        # dynamic items come last, hold at most 16 pages, and follow every static item
        first = int(np.argmax(dyn))
        assert dyn[first:].all()
        assert ((items[dyn, 2] - items[dyn, 1]) <= 16).all()


def test_plan_min_splits_and_chunk_fusion():
    """Config 5 is cut into >= 64 chunks per head (128 pages each at most); a worker running
    adjacent chunks of one head and tier carries its softmax state across them, so its
    static items never hold two adjacent pieces of the same (head, tier)."""
    sp = synth.preset(5)
    lay = workload.layout(sp, 0)
    p = _plan(sp, lay, num_workers=592, min_splits=64, max_chunk_pages=128, static_permille=1000)
    items = tg.tg_plan_items(p)
    _check_coverage(sp, lay, items)
    _check_merge_indices(items)
    for a, b in zip(items[:-1], items[1:]):
        if a[6] == b[6] and a[6] >= 0:
            assert not (a[0] == b[0] and a[5] == b[5] and a[2] == b[1])
    # the chunking still bounds dynamic items
    p = _plan(sp, lay, num_workers=592, min_splits=64, max_chunk_pages=128, static_permille=800)
    items = tg.tg_plan_items(p)
    _check_coverage(sp, lay, items)
    dyn = items[:, 6] == -1
    assert dyn.any() and ((items[dyn, 2] - items[dyn, 1]) <= 16).all()


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_plan_balances_bytes_across_workers(cfg):
    """Fully static plans: equal-cost contiguous ranges."""
    sp = synth.preset(cfg)
    lay = workload.layout(sp, 0)
    W = 592
    kw = dict(min_splits=64, max_chunk_pages=128) if cfg == 5 else {}
    p = _plan(sp, lay, num_workers=W, static_permille=1000, **kw)
    items = tg.tg_plan_items(p)
    _check_coverage(sp, lay, items)
    page_bytes = np.where(items[:, 5] & 1, 2 * (16 * sp.D + 64), 2 * 16 * sp.D * 2)
    work = np.zeros(W, np.float64)
    np.add.at(work, items[:, 6], (items[:, 2] - items[:, 1]) * page_bytes)
    assert items[:, 6].max() + 1 == W
    # equal-cost contiguous ranges: every worker within a few bf16 pages of the mean
    assert work.max() - work.mean() <= 4 * 2 * 16 * sp.D * 2
    assert work.mean() - work.min() <= 4 * 2 * 16 * sp.D * 2


def test_plan_slow_bits_validation():
    """slow_bits: 8 (default) or 4 for tiered D = 128 plans; INT4 halves the code bytes."""
    import synth
    from non_uniform_paged_flash_b200 import workload
    sp = synth.small(5)
    lay = workload.layout(sp, 0)
    B = lay.kv_len.shape[0]
    shape = tg.make_shape(B, sp.Hq, sp.Hkv, sp.D, lay.num_pages, lay.num_slow_pages, sp.page)
    kw = dict(fast_len=lay.fast_len, slow_table_len=lay.slow_table.size, num_workers=64,
              host_only=True)
    i8 = tg.tg_plan_get_info(tg.tg_plan_create(shape, lay.kv_len, lay.group_of_head,
                                               lay.group_off, **kw))["kv_bytes"]
    i4 = tg.tg_plan_get_info(tg.tg_plan_create(shape, lay.kv_len, lay.group_of_head,
                                               lay.group_off, slow_bits=4, **kw))["kv_bytes"]
    ns = int((lay.kv_len - np.minimum(lay.fast_len, lay.kv_len)).sum())
    assert i8 - i4 == ns * 2 * (sp.D // 2)
    for bad in (dict(kw, slow_bits=5), dict(num_workers=64, host_only=True, slow_bits=4)):
        with pytest.raises(tg.TGError) as ei:
            tg.tg_plan_create(shape, lay.kv_len, lay.group_of_head, lay.group_off, **bad)
        assert ei.value.status == tg.TG_EINVAL


def test_whole_heads_plan():
    """whole_heads: one item per non-empty head (every page once, no partials, no merge),
    heads placed longest first on the least-loaded worker; tiered plans ignore it."""
    rng = np.random.default_rng(61)
    B, Hq, Hkv, D = 3, 8, 4, 128
    kv = rng.integers(0, 300, (B, Hkv)).astype(np.int32)
    kv[1, 2] = 0
    goh = np.zeros(Hkv, np.int32)
    pages = -(-kv // 16)
    goff = np.array([0, int(pages.max()) * B * Hkv], np.int64)
    shape = tg.make_shape(B, Hq, Hkv, D, int(pages.sum()) + 1)
    for W in (1, 3, 64):
        p = tg.tg_plan_create(shape, kv, goh, goff, host_only=True, num_workers=W, whole_heads=True)
        info = tg.tg_plan_get_info(p)
        items = tg.tg_plan_items(p)
        nonempty = int((kv > 0).sum())
        assert info["n_items"] == nonempty and info["n_merge"] == 0 and info["n_partials"] == 0
        assert info["n_empty"] == B * Hkv - nonempty and info["n_dynamic"] == 0
        assert info["n_workers"] == min(W, nonempty)
        assert sorted(items[:, 0].tolist()) == sorted(np.nonzero(kv.reshape(-1))[0].tolist())
        for it in items:
            assert it[1] == 0 and it[2] == pages.reshape(-1)[it[0]] and it[4] == -1
        # LPT: no worker could take a head from the most-loaded one and end below it
        load = np.zeros(info["n_workers"], np.int64)
        for it in items:
            load[it[6]] += it[2]
        assert load.max() - load.min() <= pages.max()
    # tiered plans: the option is ignored (the usual split-K list)
    fl = np.minimum(kv, 40).astype(np.int32)
    shape_t = tg.make_shape(B, Hq, Hkv, D, int(pages.sum()) + 1, int(pages.sum()) + 1)
    pt = tg.tg_plan_create(shape_t, kv, goh, goff, fast_len=fl, slow_table_len=int(goff[1]),
                           host_only=True, num_workers=64, min_splits=4, whole_heads=True)
    assert tg.tg_plan_get_info(pt)["n_merge"] > 0


def test_decode_wrappers_check_sizes_and_dtypes():
    """The binding checks q / out / lse against the plan before any pointer crosses the ABI."""
    import torch
    sp = synth.small(2)
    lay = workload.layout(sp, 0)
    B = lay.kv_len.shape[0]
    shape = tg.make_shape(B, sp.Hq, sp.Hkv, sp.D, lay.num_pages)
    p = tg.tg_plan_create(shape, lay.kv_len, lay.group_of_head, lay.group_off, host_only=True,
                          num_workers=64)
    rows = B * sp.Hq
    q = torch.zeros(rows * sp.D, dtype=torch.bfloat16)
    out = torch.zeros(rows * sp.D, dtype=torch.bfloat16)
    lse = torch.zeros(rows, dtype=torch.float32)
    args = (None, None, None, None, None, None, sp.scale)
    for bad in ((q[1:], out, lse), (q, out.float(), lse), (q, out, lse[1:]), (q.float(), out, lse)):
        with pytest.raises(ValueError):
            tg.tg_ragged_paged_decode(p, bad[0], *args[:6], args[6], bad[1], bad[2])
    p32 = tg.tg_plan_create(shape, lay.kv_len, lay.group_of_head, lay.group_off, host_only=True,
                            num_workers=64, out_f32=True)
    with pytest.raises(ValueError):                   # an fp32-output plan takes fp32 out
        tg.tg_ragged_paged_decode(p32, q, *args[:6], args[6], out, lse)


def test_new_entries_reject_bad_arguments_without_a_gpu():
    """Argument checks that run before any device work: slow stream geometry, SplitZip sizes,
    host pipe on a host-only plan, INT4 append shape."""
    sp = synth.small(5)
    lay = workload.layout(sp, 0)
    B = lay.kv_len.shape[0]
    shape = tg.make_shape(B, sp.Hq, sp.Hkv, sp.D, lay.num_pages, lay.num_slow_pages, sp.page)
    ok = dict(num_workers=64, host_only=True)
    for block_pages, ring in ((0, 2), (4, 0)):
        with pytest.raises(tg.TGError) as e:
            tg.SlowStream(shape, lay.kv_len, lay.fast_len, lay.group_of_head, lay.group_off,
                          lay.slow_table, lay.slow_off, block_pages, ring, **ok)
        assert e.value.status == tg.TG_EINVAL
    bad_fl = lay.fast_len.copy()
    bad_fl[0, 0] = -1
    with pytest.raises(tg.TGError):
        tg.SlowStream(shape, lay.kv_len, bad_fl, lay.group_of_head, lay.group_off,
                      lay.slow_table, lay.slow_off, 4, 2, **ok)
    assert tg.tg_splitzip_workspace_bytes(-1) == -1
    assert tg.tg_splitzip_workspace_bytes(0) > 0
    assert tg.tg_splitzip_workspace_bytes(1 << 20) >= (1 << 20) // 8
    hp = tg.tg_plan_create(tg.make_shape(B, sp.Hq, sp.Hkv, sp.D, lay.num_pages), lay.kv_len,
                           lay.group_of_head, lay.group_off, **ok)
    with pytest.raises(tg.TGError) as e:
        tg.HostPipe(hp)
    assert e.value.status == tg.TG_EINVAL


def test_plan_rejects_unsupported_shapes_and_lengths():
    """Shapes the kernels do not serve and lengths past TG_MAX_HEAD_TOKENS are refused with
    TG_EUNSUPPORTED (a negative length with TG_EINVAL); a head of exactly the maximum plans."""
    goh = np.zeros(2, np.int32)
    goff = np.array([0, 1 << 27], np.int64)
    kv = np.array([[100, 37]], np.int32)
    ok = dict(host_only=True, num_workers=16, whole_heads=True)
    for shape in (tg.make_shape(1, 6, 2, 128, 1 << 20),      # 3 query heads per KV head
                  tg.make_shape(1, 8, 2, 96, 1 << 20),       # head dim 96
                  tg.make_shape(1, 8, 2, 128, 1 << 20, page=32)):
        with pytest.raises(tg.TGError) as e:
            tg.tg_plan_create(shape, kv, goh, goff, **ok)
        assert e.value.status == tg.TG_EUNSUPPORTED
    # 2^31 query rows: refused before any length is read (through the C entry itself; the
    # binding would first insist on B * Hkv lengths)
    big = tg.make_shape(2**28, 8, 2, 128, 1 << 20)
    opts = tg.tg_plan_opts(16, 1, 0, 1, -1, 0, 0, 0, 0, 0, 0, 0, 8, 1)
    h = ctypes.c_void_p()
    kvc, gohc, goffc = (np.ascontiguousarray(kv), np.ascontiguousarray(goh),
                        np.ascontiguousarray(goff))
    assert tg._lib().tg_plan_create(ctypes.byref(big), kvc.ctypes.data, None, gohc.ctypes.data,
                                    goffc.ctypes.data, 1, 0, ctypes.byref(opts),
                                    ctypes.byref(h)) == tg.TG_EUNSUPPORTED
    assert not h.value
    with pytest.raises(ValueError):                  # the binding's own size check
        tg.tg_plan_create(big, kv, goh, goff, **ok)
    shape = tg.make_shape(1, 8, 2, 128, 1 << 26)
    for bad, status in ((tg.TG_MAX_HEAD_TOKENS + 1, tg.TG_EUNSUPPORTED),
                        (2**31 - 1, tg.TG_EUNSUPPORTED), (-1, tg.TG_EINVAL)):
        with pytest.raises(tg.TGError) as e:
            tg.tg_plan_create(shape, np.array([[100, bad]], np.int32), goh, goff, **ok)
        assert e.value.status == status
    p = tg.tg_plan_create(shape, np.array([[100, tg.TG_MAX_HEAD_TOKENS]], np.int32), goh, goff, **ok)
    info = tg.tg_plan_get_info(p)
    assert info["n_items"] == 2
    assert info["kv_bytes"] == (100 + tg.TG_MAX_HEAD_TOKENS) * 2 * 128 * 2


def test_binding_checks_host_array_sizes():
    """Host arrays whose size the C side infers from the shape are checked before the call
    (a short array would otherwise be read past its end)."""
    shape = tg.make_shape(2, 8, 2, 128, 1024)
    kv = np.array([[40, 17], [3, 90]], np.int32)
    goh = np.zeros(2, np.int32)
    goff = np.array([0, 64], np.int64)
    ok = dict(host_only=True, num_workers=8)
    tg.tg_plan_destroy(tg.tg_plan_create(shape, kv, goh, goff, **ok))
    for bad in (dict(kv_len=kv[:1]), dict(group_of_head=goh[:1]), dict(group_off=goff[:1]),
                dict(fast_len=np.zeros(3, np.int32))):
        args = dict(kv_len=kv, group_of_head=goh, group_off=goff)
        args.update(bad)
        with pytest.raises(ValueError):
            tg.tg_plan_create(shape, args["kv_len"], args["group_of_head"], args["group_off"],
                              fast_len=args.get("fast_len"), **ok)
    table = np.arange(16, dtype=np.int32)
    with pytest.raises(ValueError):
        tg.tg_plan_create_cascade(shape, kv, goh, goff, table, np.zeros(3, np.int64), **ok)
    with pytest.raises(ValueError):
        tg.tg_alloc_create_ordered(10, 16, np.arange(9))
    cnt = np.array([[2, 1], [0, 3]], np.int32)
    with pytest.raises(ValueError):
        tg.tg_build_group_tables(cnt, np.zeros(3, np.int32), 1, np.arange(6))
    with pytest.raises(ValueError):
        tg.tg_build_group_tables(cnt, np.zeros(2, np.int32), 1, np.arange(5))   # 6 page ids needed
    t, off, g = tg.tg_build_group_tables(cnt, np.zeros(2, np.int32), 1, np.arange(6))
    assert g[-1] == 2 * 2 * 3


def test_allocator_outputs_sized_with_its_own_page():
    """The binding sizes segment and reservation outputs with the allocator's page (a larger
    page argument would under-size them); a page argument that disagrees is refused."""
    a = tg.tg_alloc_create_ordered(64, 8)
    try:
        sid, ids = tg.tg_share_segment(a, 40, 2)               # 5 full 8-token pages per head
        assert ids.shape == (2, 5) and len(np.unique(ids)) == 10
        with pytest.raises(ValueError):
            tg.tg_share_segment(a, 40, 2, 16)
        r = tg.tg_reserve(a, 0, [41, 40], [sid])               # 40 shared + 1 private token
        assert r.size == 5 + 1 + 5 and tg.tg_alloc_free_pages(a) == 64 - 10 - 1
        with pytest.raises(ValueError):
            tg.tg_reserve(a, 1, [8], (), 16)
    finally:
        tg.tg_alloc_destroy(a)


def test_splitzip_buffers_are_size_checked():
    """Every SplitZip buffer is checked against n before a kernel could index past its end."""
    import torch
    n, cap = 100, 10
    ok = dict(src=torch.zeros(n, dtype=torch.int16), codebook=torch.zeros(16, dtype=torch.uint8),
              sm=torch.zeros(n, dtype=torch.uint8), codes=torch.zeros(50, dtype=torch.uint8),
              esc_pos=torch.zeros(cap, dtype=torch.int64), esc_exp=torch.zeros(cap, dtype=torch.uint8),
              n_esc=torch.zeros(1, dtype=torch.int64),
              workspace=torch.zeros(tg.tg_splitzip_workspace_bytes(n), dtype=torch.uint8))
    short = dict(src=ok["src"][:n - 1], codebook=ok["codebook"][:15], sm=ok["sm"][:n - 1],
                 codes=ok["codes"][:49], esc_exp=ok["esc_exp"][:cap - 1], n_esc=torch.zeros(0, dtype=torch.int64),
                 workspace=ok["workspace"][:-1])
    for name, t in short.items():
        args = dict(ok, **{name: t})
        with pytest.raises(ValueError, match=name):
            tg.tg_splitzip_encode(n, args["src"], args["codebook"], args["sm"], args["codes"],
                                  args["esc_pos"], args["esc_exp"], args["n_esc"], args["workspace"])
    with pytest.raises(ValueError, match="dst"):
        tg.tg_splitzip_decode(n, ok["codebook"], ok["sm"], ok["codes"], ok["esc_pos"], ok["esc_exp"],
                              ok["n_esc"], torch.zeros(n - 1, dtype=torch.int16))
    with pytest.raises(ValueError, match="sm"):
        tg.tg_splitzip_decode(n, ok["codebook"], short["sm"], ok["codes"], ok["esc_pos"], ok["esc_exp"],
                              ok["n_esc"], torch.zeros(n, dtype=torch.int16))


def test_quantizer_and_merge_outputs_are_size_checked():
    import torch
    src = torch.zeros((10, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="codes"):
        tg.tg_quantize_int8(src, torch.zeros(10 * 128 - 1, dtype=torch.int8), torch.zeros(10))
    with pytest.raises(ValueError, match="scale"):
        tg.tg_quantize_int8(src, torch.zeros(10 * 128, dtype=torch.int8), torch.zeros(9))
    with pytest.raises(ValueError, match="packed"):
        tg.tg_quantize_int4(src, torch.zeros(10 * 64 - 1, dtype=torch.uint8), torch.zeros(10))
    off = torch.tensor([0, 2, 3], dtype=torch.int64)
    po, pl = torch.zeros((3, 128)), torch.zeros(3)
    with pytest.raises(ValueError, match="out"):
        tg.tg_lse_merge(off, po, pl, torch.zeros((1, 128), dtype=torch.bfloat16), torch.zeros(2))
    with pytest.raises(ValueError, match="lse"):
        tg.tg_lse_merge(off, po, pl, torch.zeros((2, 128), dtype=torch.bfloat16), torch.zeros(1))
