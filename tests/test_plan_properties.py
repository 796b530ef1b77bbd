"""Planner invariants over random shapes, lengths and options (hypothesis; host-only plans,
no GPU): every page of every (sequence, KV head) and tier is covered by exactly one item;
a head with one item writes the final output, a split head's items take consecutive partial
slots and one merge index; empty heads are reported; dynamic items come last."""
import numpy as np
from hypothesis import given, settings, strategies as st

import non_uniform_paged_flash_b200 as tg


@st.composite
def plans(draw):
    B = draw(st.integers(1, 5))
    Hkv = draw(st.sampled_from([1, 2, 4, 8]))
    G = draw(st.sampled_from([1, 2, 4, 8]))
    D = draw(st.sampled_from([64, 128]))
    tiered = draw(st.booleans())
    if tiered:
        D = 128
    kv = np.array(draw(st.lists(st.integers(0, 700), min_size=B * Hkv, max_size=B * Hkv)), np.int32)
    fl = (np.array(draw(st.lists(st.integers(0, 300), min_size=B * Hkv, max_size=B * Hkv)), np.int32)
          if tiered else None)
    opts = dict(num_workers=draw(st.integers(1, 300)),
                min_splits=draw(st.integers(1, 9)),
                max_chunk_pages=draw(st.sampled_from([0, 1, 3, 16])),
                static_permille=draw(st.sampled_from([0, 300, 850, 1000])),
                dyn_chunk_pages=draw(st.sampled_from([0, 1, 4, 16])),
                whole_heads=draw(st.booleans()) and not tiered,
                slow_bits=draw(st.sampled_from([8, 4])) if tiered else 8)
    return B, Hkv, G, D, kv.reshape(B, Hkv), None if fl is None else fl.reshape(B, Hkv), opts


@settings(max_examples=250, deadline=None)
@given(plans())
def test_plan_invariants(case):
    B, Hkv, G, D, kv, fl, opts = case
    pages_f = -(-(np.minimum(fl, kv) if fl is not None else np.zeros_like(kv)) // 16)
    pages_s = -(-(kv - (np.minimum(fl, kv) if fl is not None else 0)) // 16)
    total = int(pages_s.sum() + pages_f.sum())
    shape = tg.make_shape(B, G * Hkv, Hkv, D, total + 1, total + 1 if fl is not None else 0)
    goff = np.array([0, int(max(1, (pages_f if fl is not None else pages_s).max())) * B * Hkv],
                    np.int64)
    p = tg.tg_plan_create(shape, kv, np.zeros(Hkv, np.int32), goff, fast_len=fl,
                          slow_table_len=int(pages_s.max(initial=1)) * B * Hkv if fl is not None else 0,
                          host_only=True, **opts)
    info = tg.tg_plan_get_info(p)
    items = tg.tg_plan_items(p)
    assert info["n_items"] == len(items)
    seen = {}
    for bh, pb, pe, tt, slot, tier, worker, mi in items:
        assert 0 <= pb < pe
        for pg in range(pb, pe):
            key = (int(bh), int(tier), pg)
            assert key not in seen, key
            seen[key] = True
    want = 0
    for bh in range(B * Hkv):
        ns = int(pages_s.reshape(-1)[bh])                  # the untiered pages when not tiered
        nf = int(pages_f.reshape(-1)[bh]) if fl is not None else 0
        if fl is None:
            assert all((bh, 0, pg) in seen for pg in range(ns))
        else:
            assert all((bh, 1, pg) in seen for pg in range(ns))
            assert all((bh, 0, pg) in seen for pg in range(nf))
        want += ns + nf
    assert len(seen) == want
    # slots and merge indices
    heads = {}
    for row in items:
        heads.setdefault(int(row[0]), []).append(row)
    merge_idx = set()
    for bh, rows in heads.items():
        if len(rows) == 1:
            assert rows[0][4] == -1 and rows[0][7] == -1
        else:
            slots = sorted(int(r[4]) for r in rows)
            assert slots == list(range(slots[0], slots[0] + len(rows)))
            mis = {int(r[7]) for r in rows}
            assert len(mis) == 1
            merge_idx |= mis
    assert sorted(merge_idx) == list(range(len(merge_idx))) and info["n_merge"] == len(merge_idx)
    assert info["n_empty"] == int((kv == 0).sum())
    dyn = items[:, 6] == -1
    assert info["n_dynamic"] == int(dyn.sum())
    if dyn.any():
        assert dyn[int(np.argmax(dyn)):].all()
    if opts["whole_heads"]:
        assert info["n_merge"] == 0 and len(items) == int((kv > 0).sum())


def test_whole_head_plans_of_short_heads_take_the_lean_kernel():
    """Whole-head bf16 plans whose heads hold at most 64 pages report the lean kernel's launch
    (one CTA of 256 threads per (sequence, KV head), no ring, no shared-memory carve-out); longer
    heads, split plans and tiered plans keep the pipelined kernel."""
    import non_uniform_paged_flash_b200 as tg

    def info(kv, **kw):
        kv = np.asarray(kv, np.int32)
        B, H = kv.shape
        shape = tg.make_shape(B, 4 * H, H, 128, 1 << 16, 1 << 12 if "fast_len" in kw else 0)
        plan = tg.tg_plan_create(shape, kv, np.zeros(H, np.int32), np.array([0, 1 << 20], np.int64),
                                 host_only=True, **kw)
        return tg.tg_plan_get_info(plan)

    # lean: one CTA per (sequence, KV head), the empty head included
    lean = info([[1024, 0, 17], [1, 999, 64]], whole_heads=True)
    assert (lean["grid"], lean["block"], lean["stages"], lean["smem_bytes"]) == (6, 256, 0, 0)
    assert lean["n_merge"] == 0 and lean["n_empty"] == 1
    # a head of 65 pages: the pipelined kernel, its 2 whole heads on one CTA of 4 workers
    long_ = info([[1025, 10]], whole_heads=True)
    assert long_["grid"] == 1 and long_["n_workers"] == 2
    split = info([[1024, 10]])
    assert split["block"] == 4 * 64 and split["grid"] == -(-split["n_workers"] // 4)
    tiered = info([[1024, 10]], whole_heads=True, fast_len=np.array([[100, 10]], np.int32),
                  slow_table_len=1 << 10)
    assert tiered["block"] == 6 * 64
