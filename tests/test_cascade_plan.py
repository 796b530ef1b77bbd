"""Host logic of the prefix-aware cascade plan (no GPU): every (sequence, KV head, page) is read
exactly once, by one cascade unit (a run of pages several rows share at the same positions) or
one ordinary item; the rows of a unit really hold the same pages there; each head's partials
form one contiguous merge range, cascade runs first.
"""
import numpy as np
import pytest

import non_uniform_paged_flash_b200 as tg
import synth
from non_uniform_paged_flash_b200 import workload


def _cascade_plan(B, Hq, Hkv, D, num_pages, kv_len, table, head_off, min_readers=2, **kw):
    shape = tg.make_shape(B, Hq, Hkv, D, num_pages)
    goh = np.zeros(Hkv, np.int32)
    goff = np.array([0, max(table.size, 1)], np.int64)
    return tg.tg_plan_create_cascade(shape, kv_len, goh, goff, table, head_off,
                                     min_readers=min_readers, host_only=True, **kw)


def check_cascade(plan, B, Hq, Hkv, kv_len, table, head_off, min_readers=2):
    G = Hq // Hkv
    kv = np.asarray(kv_len).reshape(-1).astype(np.int64)
    hoff = np.asarray(head_off).reshape(-1)
    meta, readers, slots = tg.tg_plan_cascade_units(plan)
    items = tg.tg_plan_items(plan)
    seen = {}
    partials = {}
    runs = {}
    for (h, pb, pe, nr), rd, sl in zip(meta, readers, slots):
        assert 0 <= pb < pe and 1 <= nr <= tg.CASCADE_ROWS // G
        assert (rd[nr:] == -1).all() and (sl[nr:] == -1).all()
        rows = rd[:nr]
        for b in rows:
            bh = int(b) * Hkv + int(h)
            assert kv[bh] >= pe * 16, "a run holds full pages only"
            np.testing.assert_array_equal(table[hoff[bh] + pb: hoff[bh] + pe],
                                          table[hoff[int(rows[0]) * Hkv + h] + pb: hoff[int(rows[0]) * Hkv + h] + pe])
            for p in range(pb, pe):
                assert (bh, p) not in seen, (bh, p)
                seen[(bh, p)] = "cascade"
        for b, s in zip(rows, sl[:nr]):
            partials.setdefault(int(b) * Hkv + int(h), []).append(("c", int(s)))
        runs.setdefault((int(h), int(pb), int(pe)), set()).update(int(b) for b in rows)
    for (h, pb, pe), rows in runs.items():
        assert len(rows) >= max(2, min_readers)
    for bh, pb, pe, tt, slot, tier, worker, mi in items:
        assert tier == 0
        for p in range(pb, pe):
            assert (bh, p) not in seen, (bh, p)
            seen[(bh, p)] = "item"
        partials.setdefault(int(bh), []).append(("i", int(slot)))
    want = {(bh, p) for bh in range(kv.size) for p in range(-(-kv[bh] // 16))}
    assert set(seen) == want
    all_slots = []
    for bh, lst in partials.items():
        s = [x for _, x in lst]
        if len(lst) == 1 and lst[0][0] == "i":
            assert s == [-1]
            continue
        assert all(x >= 0 for x in s)
        c = sorted(x for k, x in lst if k == "c")
        i = sorted(x for k, x in lst if k == "i")
        merged = c + i
        assert merged == list(range(merged[0], merged[0] + len(merged))), "one contiguous range"
        all_slots += merged
    assert len(all_slots) == len(set(all_slots))
    info = tg.tg_plan_get_info(plan)
    assert info["n_partials"] == len(all_slots)
    return meta, items


@pytest.mark.parametrize("full", [False, True])
def test_prefix_config_runs(full):
    """Config 4: per KV head one run of the system pages read by every sequence, and one run
    of each document's full pages read by the sequences on it."""
    sp = synth.preset(4) if full else synth.small(4)
    lay = workload.layout(sp, 0)
    B = lay.kv_len.shape[0]
    plan = _cascade_plan(B, sp.Hq, sp.Hkv, sp.D, lay.num_pages, lay.kv_len, lay.table,
                         lay.head_off)
    meta, items = check_cascade(plan, B, sp.Hq, sp.Hkv, lay.kv_len, lay.table, lay.head_off)
    sys_pages = sp.sys_tokens // 16
    doc_pages = sp.doc_tokens // 16
    doc, _ = synth.prefix_layout(sp)
    per = tg.CASCADE_ROWS // (sp.Hq // sp.Hkv)
    for h in range(sp.Hkv):
        m = meta[meta[:, 0] == h]
        sysu = m[(m[:, 1] == 0) & (m[:, 2] == sys_pages)]
        assert sysu[:, 3].sum() == B and len(sysu) == -(-B // per)
        docu = m[(m[:, 1] == sys_pages) & (m[:, 2] == sys_pages + doc_pages)]
        readers = sorted(np.bincount(doc, minlength=sp.n_docs)[np.bincount(doc, minlength=sp.n_docs) >= 2])
        assert docu[:, 3].sum() == sum(readers)
    # the private items start after the deepest run of each row
    assert (items[:, 1] >= sys_pages + doc_pages).all()


def _random_tree_layout(rng, B, Hkv, n_roots=2, depth=3, fan=3):
    """Rows built from a random prefix tree of page runs (per KV head its own tree), then a
    private tail (which may end in a partial page); a few rows repeat a shared page at another
    position, and a few are exactly a shared path (no private page)."""
    next_pid = [0]

    def new_pages(n):
        out = list(range(next_pid[0], next_pid[0] + n))
        next_pid[0] += n
        return out

    rows = {}
    for h in range(Hkv):
        paths = []

        def grow(prefix, d):
            paths.append(prefix)
            if d == depth:
                return
            for _ in range(int(rng.integers(1, fan + 1))):
                grow(prefix + new_pages(int(rng.integers(1, 5))), d + 1)

        for _ in range(n_roots):
            grow(new_pages(int(rng.integers(1, 6))), 1)
        for b in range(B):
            path = paths[int(rng.integers(0, len(paths)))]
            kind = rng.random()
            if kind < 0.1:
                toks = len(path) * 16                          # exactly a shared path
                pages = list(path)
            else:
                extra = int(rng.integers(1, 60))
                pages = list(path) + new_pages(-(-extra // 16))
                toks = len(path) * 16 + extra
                if kind < 0.2 and len(path) > 1:
                    pages = pages[:1] + [path[-1]] + pages[1:-1]  # shared page, other position
                    toks = min(toks, len(pages) * 16)
            rows[(b, h)] = (pages, toks)
    table, head_off, kv = [], np.zeros((B, Hkv), np.int64), np.zeros((B, Hkv), np.int32)
    for b in range(B):
        for h in range(Hkv):
            pages, toks = rows[(b, h)]
            head_off[b, h] = len(table)
            table += pages
            kv[b, h] = toks
    return np.array(table, np.int32), head_off, kv, next_pid[0]


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_random_prefix_trees(seed, G):
    rng = np.random.default_rng(100 + seed)
    B, Hkv = int(rng.integers(2, 90)), int(rng.integers(1, 4))
    table, head_off, kv, P = _random_tree_layout(rng, B, Hkv)
    for min_readers in (2, 5):
        plan = _cascade_plan(B, G * Hkv, Hkv, 128, P, kv, table, head_off, min_readers=min_readers,
                             num_workers=int(rng.integers(1, 300)))
        check_cascade(plan, B, G * Hkv, Hkv, kv, table, head_off, min_readers)


def test_cascade_rejects_rows_outside_the_table():
    table = np.arange(4, dtype=np.int32)
    with pytest.raises(tg.TGError) as e:
        _cascade_plan(1, 4, 1, 128, 4, np.array([[80]], np.int32), table, np.array([[0]], np.int64))
    assert e.value.status == tg.TG_EINVAL


def test_no_sharing_gives_no_units():
    sp = synth.small(2)
    lay = workload.layout(sp, 0)
    plan = _cascade_plan(sp.B, sp.Hq, sp.Hkv, sp.D, lay.num_pages, lay.kv_len, lay.table,
                         lay.head_off)
    assert tg.tg_plan_get_info(plan)["n_cascade"] == 0
    check_cascade(plan, sp.B, sp.Hq, sp.Hkv, lay.kv_len, lay.table, lay.head_off)
