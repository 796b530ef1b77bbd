"""The allocator's own seeded shuffle (tg_alloc_create): the initial free list is Durstenfeld's
Fisher-Yates shuffle driven by SplitMix64 from the seed. Pinned to the generator's published
seed-0 outputs on tiny pools, and to the independent input generator's free order (synth,
plain C) on large ones; the allocator hands pages out in free-list order, which a one-head
reservation of the whole pool (page = 1 token) reads back."""
import numpy as np
import pytest

import non_uniform_paged_flash_b200 as tg
import synth


def _free_list(n, seed):
    a = tg.tg_alloc_create(n, 1, seed)
    try:
        ids, counts = tg.tg_reserve(a, 0, [n], (), 1, with_counts=True)
        assert counts.tolist() == [n] and tg.tg_alloc_free_pages(a) == 0
        return ids
    finally:
        tg.tg_alloc_destroy(a)


def test_seed_zero_against_published_splitmix64_outputs():
    # SplitMix64 seeded with 0 first outputs 0xe220a8397b1dcdaf, 0x6e789e6aa1b965f4,
    # 0x06c45d188009454f (Steele, Lea & Flood 2014; the generator's common test vector).
    # n = 3: i = 2 swaps with 0x...cdaf mod 3 = 1 -> [0, 2, 1]; i = 1 with 0x...65f4 mod 2 = 0
    # -> [2, 0, 1]. n = 4: i = 3 with 0x...cdaf mod 4 = 3 (no move); i = 2 with
    # 0x...65f4 mod 3 = 0 -> [2, 1, 0, 3]; i = 1 with 0x...454f mod 2 = 1 (no move).
    assert _free_list(1, 0).tolist() == [0]
    assert _free_list(2, 0).tolist() == [0, 1]
    assert _free_list(3, 0).tolist() == [2, 0, 1]
    assert _free_list(4, 0).tolist() == [2, 1, 0, 3]


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("slow", [False, True])
def test_library_shuffle_equals_the_input_generators(cfg, slow):
    sp = synth.preset(cfg)
    for n, layer in ((1, 0), (97, 0), (65536, 1), (743311, 17)):
        want = synth.free_order(sp, n, layer, slow=slow)
        got = _free_list(n, synth.free_order_seed(sp, layer, slow=slow))
        np.testing.assert_array_equal(got, want)


def test_every_seed_gives_a_permutation():
    for seed in (0, 1, 2 ** 63, 2 ** 64 - 1, 0x7A4E0003):
        ids = _free_list(1000, seed)
        assert sorted(ids.tolist()) == list(range(1000))


def test_reserve_reports_each_heads_page_count():
    """tg_reserve's per-head counts: shared full pages plus ceil(private tokens / page)."""
    a = tg.tg_alloc_create(1000, 16, 5)
    try:
        sid, seg = tg.tg_share_segment(a, 50, 2, 16)                 # 3 full pages per head
        ids, counts = tg.tg_reserve(a, 7, [50, 80], (sid,), 16, with_counts=True)
        assert counts.tolist() == [3 + 1, 3 + 2]                       # 2 and 32 private tokens
        assert ids.size == counts.sum()
        assert ids[:3].tolist() == seg[0].tolist() and ids[4:7].tolist() == seg[1].tolist()
        ids, counts = tg.tg_reserve(a, 8, [0, 1, 16, 17], (), 16, with_counts=True)
        assert counts.tolist() == [0, 1, 1, 2]
    finally:
        tg.tg_alloc_destroy(a)
