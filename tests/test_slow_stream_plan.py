"""Host logic of the streamed slow tier (no GPU): the blocks a tg_slow_stream copies and the
tokens of every (sequence, KV head) in each, against a direct count from the layout's own
INT8-tier table; blocks without a retained token are skipped; bad page ids are rejected.
"""
from dataclasses import replace

import numpy as np
import pytest

import non_uniform_paged_flash_b200 as tg
import synth
from non_uniform_paged_flash_b200 import workload


def _count(lay, block_pages):
    """tokens[block][bh] counted page by page from the slow table."""
    nsp = lay.num_slow_pages
    J = (nsp + block_pages - 1) // block_pages
    BH = lay.kv_len.size
    tok = np.zeros((J, BH), np.int64)
    kv, fl = lay.kv_len.reshape(-1), lay.fast_len.reshape(-1)
    for bh in range(BH):
        ns = kv[bh] - min(fl[bh], kv[bh])
        for t in range((ns + 15) // 16):
            pid = lay.slow_table[lay.slow_off.reshape(-1)[bh] + t]
            tok[pid // block_pages, bh] += min(16, ns - 16 * t)
    return tok


def _stream(lay, sp, block_pages, ring=2):
    B = lay.kv_len.shape[0]
    shape = tg.make_shape(B, sp.Hq, sp.Hkv, sp.D, lay.num_pages, lay.num_slow_pages, sp.page)
    return tg.SlowStream(shape, lay.kv_len, lay.fast_len, lay.group_of_head, lay.group_off,
                         lay.slow_table, lay.slow_off, block_pages, ring, num_workers=64,
                         host_only=True)


@pytest.mark.parametrize("block_pages", [1, 3, 7, 64, 1 << 20])
def test_blocks_partition_the_slow_tier(block_pages):
    sp = synth.small(5)
    lay = workload.layout(sp, 0)
    ss = _stream(lay, sp, block_pages)
    first, pages, tokens = ss.blocks()
    want = _count(lay, block_pages)
    used = np.nonzero(want.sum(1))[0]
    np.testing.assert_array_equal(first, used * block_pages)
    np.testing.assert_array_equal(pages, np.minimum(block_pages, lay.num_slow_pages - first))
    np.testing.assert_array_equal(tokens, want[used])
    kv, fl = lay.kv_len.reshape(-1), lay.fast_len.reshape(-1)
    np.testing.assert_array_equal(tokens.sum(0), kv - np.minimum(fl, kv))


def test_unused_pages_make_no_block_and_all_fast_heads_none():
    sp = replace(synth.small(5), occupancy_num=3, occupancy_den=1)   # pool 3x the used pages
    lay = workload.layout(sp, 0)
    ss = _stream(lay, sp, 5)
    first, pages, tokens = ss.blocks()
    assert (tokens.sum(1) > 0).all()
    assert len(first) < (lay.num_slow_pages + 4) // 5
    lay2 = replace(lay, fast_len=lay.kv_len.copy())   # every token in the fast tier
    ss2 = _stream(lay2, sp, 5)
    assert ss2.blocks()[0].size == 0


def test_bad_page_id_is_rejected():
    sp = synth.small(5)
    lay = workload.layout(sp, 0)
    bad = lay.slow_table.copy()
    bad[3] = lay.num_slow_pages
    with pytest.raises(tg.TGError) as ei:
        _stream(replace(lay, slow_table=bad), sp, 4)
    assert ei.value.status == tg.TG_EINVAL


def test_blocks_do_not_depend_on_code_width():
    """INT4 and INT8 slow tiers stream the same blocks and tokens (only the bytes differ)."""
    sp = synth.small(5)
    lay = workload.layout(sp, 0)
    B = lay.kv_len.shape[0]
    shape = tg.make_shape(B, sp.Hq, sp.Hkv, sp.D, lay.num_pages, lay.num_slow_pages, sp.page)
    got = []
    for bits in (8, 4):
        ss = tg.SlowStream(shape, lay.kv_len, lay.fast_len, lay.group_of_head, lay.group_off,
                           lay.slow_table, lay.slow_off, 7, 2, num_workers=64, host_only=True,
                           slow_bits=bits)
        got.append(ss.blocks())
    for a, b in zip(*got):
        np.testing.assert_array_equal(a, b)


def test_algorithmic_bytes_int4_closed_form():
    """Per slow token-head 2 (D/2 + 4) bytes for INT4 and 2 (D + 4) for INT8; fast 4 D."""
    sp = synth.small(5)
    lay = workload.layout(sp, 0)
    kv = lay.kv_len.astype(np.int64)
    f = np.minimum(lay.fast_len.astype(np.int64), kv)
    for bits, row in ((8, sp.D), (4, sp.D // 2)):
        alg = workload.algorithmic_bytes(replace(sp, slow_bits=bits), lay)
        assert alg["kv"] == int((kv - f).sum()) * 2 * (row + 4) + int(f.sum()) * 4 * sp.D
