"""Budget-reservation allocator against the oracle's layout over random batches (hypothesis):
random retained lengths, shared segments, per-sequence segment chains (with absent entries),
shuffled free orders and page sizes; the library's page ids and segment pages must equal the
oracle's bit for bit, and a pool one page short must be refused with nothing taken."""
import numpy as np
from hypothesis import given, settings, strategies as st

import non_uniform_paged_flash_b200 as tg
import oracle


@st.composite
def batches(draw):
    page = draw(st.sampled_from([16, 8, 1, 5]))
    B = draw(st.integers(1, 6))
    H = draw(st.integers(1, 4))
    n_segs = draw(st.integers(0, 3))
    segs = [draw(st.integers(0, 6 * page)) for _ in range(n_segs)]
    chain_len = draw(st.integers(0, 2)) if n_segs else 0
    chain = np.array([[draw(st.integers(-1, n_segs - 1)) for _ in range(chain_len)] for _ in range(B)],
                     dtype=np.int64).reshape(B, chain_len)
    shared = np.array([sum(segs[c] // page * page for c in row if c >= 0) for row in chain]
                      if chain_len else [0] * B, dtype=np.int64)
    extra = np.array([[draw(st.integers(0, 5 * page)) for _ in range(H)] for _ in range(B)], dtype=np.int64)
    kv = (shared[:, None] + extra).astype(np.int32)
    seg_pages = sum(H * (s // page) for s in segs)
    priv = int(((kv - shared[:, None] + page - 1) // page).sum())
    exact = seg_pages + priv
    slack = draw(st.integers(0, 4))
    seed = draw(st.integers(0, 2**32 - 1))
    return page, segs, chain, kv, exact, slack, seed


def _lib_layout(num_pages, order, kv, segs, chain, page):
    a = tg.tg_alloc_create_ordered(num_pages, page, order)
    try:
        seg_ids, seg_pages = [], []
        for s in segs:
            sid, ids = tg.tg_share_segment(a, s, kv.shape[1], page)
            seg_ids.append(sid)
            seg_pages.append(ids.reshape(-1))
        out = []
        for b in range(kv.shape[0]):
            pre = [seg_ids[c] if c >= 0 else -1 for c in chain[b]]
            out.append(tg.tg_reserve(a, b, kv[b], pre, page))
        free_left = tg.tg_alloc_free_pages(a)
        return (np.concatenate(out) if out else np.zeros(0, np.int32),
                np.concatenate(seg_pages) if seg_pages else np.zeros(0, np.int32), free_left)
    finally:
        tg.tg_alloc_destroy(a)


@settings(max_examples=300, deadline=None)
@given(batches())
def test_allocator_layout_equals_oracle(case):
    page, segs, chain, kv, exact, slack, seed = case
    num_pages = max(1, exact + slack)
    order = np.random.default_rng(seed).permutation(num_pages).astype(np.int32)
    ids, segp, free_left = _lib_layout(num_pages, order, kv, segs, chain, page)
    oids, ocount, osegp = oracle.reservation_layout(num_pages, order, page, kv, segs,
                                                    chain if chain.shape[1] else None)
    np.testing.assert_array_equal(ids, oids)
    np.testing.assert_array_equal(segp, osegp)
    assert free_left == num_pages - exact
    assert int(np.asarray(ocount).sum()) == ids.size


@settings(max_examples=100, deadline=None)
@given(batches())
def test_pool_one_page_short_is_refused_without_taking_pages(case):
    page, segs, chain, kv, exact, _, seed = case
    if exact < 2:
        return
    num_pages = exact - 1
    order = np.random.default_rng(seed).permutation(num_pages).astype(np.int32)
    a = tg.tg_alloc_create_ordered(num_pages, page, order)
    try:
        seg_ids = []
        for s in segs:
            try:
                sid, _ = tg.tg_share_segment(a, s, kv.shape[1], page)
            except tg.TGError as e:
                assert e.status == tg.TG_ENOSPC
                return                                   # the segments alone do not fit
            seg_ids.append(sid)
        refused = False
        for b in range(kv.shape[0]):
            before = tg.tg_alloc_free_pages(a)
            pre = [seg_ids[c] if c >= 0 else -1 for c in chain[b]]
            try:
                tg.tg_reserve(a, b, kv[b], pre, page)
            except tg.TGError as e:
                assert e.status == tg.TG_ENOSPC
                assert tg.tg_alloc_free_pages(a) == before   # nothing taken
                refused = True
                break
        assert refused
    finally:
        tg.tg_alloc_destroy(a)


@settings(max_examples=200, deadline=None)
@given(st.integers(0, 7), st.integers(1, 9), st.integers(1, 9), st.integers(0, 12), st.integers(0, 2**32 - 1))
def test_group_tables_equal_oracle(B, H, G, max_pages, seed):
    """Group page tables (any group map, empty groups included) against the oracle's."""
    G = min(G, H)
    rng = np.random.default_rng(seed)
    cnt = rng.integers(0, max_pages + 1, (B, H)).astype(np.int32)
    goh = rng.integers(0, G, H).astype(np.int32)
    ids = rng.permutation(int(cnt.sum()) + 2)[: int(cnt.sum())].astype(np.int32)
    t, off, goff = tg.tg_build_group_tables(cnt, goh, G, ids)
    ot, ooff, ogoff = oracle.group_tables(goh, G, ids, cnt)
    np.testing.assert_array_equal(t, ot)
    np.testing.assert_array_equal(goff, ogoff)
    np.testing.assert_array_equal(off, ooff)


@settings(max_examples=200, deadline=None)
@given(st.lists(st.integers(0, 10**9), min_size=0, max_size=60), st.integers(1, 9))
def test_placement_equals_oracle(seq_bytes, n_gpus):
    """Ahead-of-time placement (ties included) against the oracle's LPT."""
    b = np.asarray(seq_bytes, dtype=np.int64)
    np.testing.assert_array_equal(tg.tg_place_sequences(b, n_gpus), oracle.place_sequences(b, n_gpus))


@settings(max_examples=200, deadline=None)
@given(st.lists(st.tuples(st.integers(0, 2**31 - 1), st.integers(0, 1_000_000)), min_size=1, max_size=40),
       st.integers(1, 8))
def test_lengths_and_groups_equal_oracle(pairs, n_groups):
    """Retained lengths (full int32 range of lengths) and budget groups against the oracle's."""
    full = np.array([p[0] for p in pairs], dtype=np.int32)
    ratio = np.array([p[1] for p in pairs], dtype=np.int32)
    np.testing.assert_array_equal(tg.tg_retained_lengths(full, ratio),
                                  oracle.retained_lengths(full, ratio))
    G = min(n_groups, len(pairs))
    np.testing.assert_array_equal(tg.tg_budget_groups(ratio, G), oracle.budget_groups(ratio, G))
