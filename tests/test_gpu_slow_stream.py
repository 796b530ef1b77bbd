"""GPU parity of the streamed slow tier: the INT8 tier read from pinned host memory block by
block through the HBM ring gives the fp64 oracle's tiered result (out <= 2e-2, lse <= 1e-3),
for one block, many blocks, a ring of one, unused pool pages and repeated steps; the fp32
output plans it is built on match the bf16 call; pageable host memory is rejected.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import non_uniform_paged_flash_b200 as tg
import synth
from non_uniform_paged_flash_b200 import workload
from tests import _oracle_side as ors

pytestmark = pytest.mark.gpu


def _check(db, sp, lay):
    ol = ors.layout(sp, 0)
    ors.assert_same_layout(lay, ol)
    ref_out, ref_lse = ors.reference(sp, ol, 0)
    out = db.out.float().cpu().numpy().reshape(-1, sp.D)
    lse = db.lse.cpu().numpy().reshape(-1)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.abs(out - ref_out).max() <= 2e-2
    assert np.abs(lse[fin] - ref_lse[fin]).max() <= 1e-3


@pytest.mark.parametrize("block_pages,ring", [(1 << 20, 2), (64, 3), (7, 2), (5, 1)])
def test_streamed_tier_matches_oracle(block_pages, ring):
    sp = synth.small(5)
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, min_splits=8, max_chunk_pages=16)
    host = db.host_slow_tier()
    ss = db.slow_stream(block_pages, ring, min_splits=4)
    for step in range(3):   # ring slots are reused across steps
        db.out.zero_()
        db.run_streamed(ss, host)
        torch.cuda.synchronize()
        assert ss.status() == tg.TG_OK
        _check(db, sp, lay)
        if step == 0:
            first = (db.out.clone(), db.lse.clone())
        else:
            assert torch.equal(db.out, first[0]) and torch.equal(db.lse, first[1])


def test_streamed_tier_with_unused_pool_pages():
    sp = replace(synth.small(5), occupancy_num=3, occupancy_den=1)
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, min_splits=8, max_chunk_pages=16)
    ss = db.slow_stream(9, 2)
    db.run_streamed(ss, db.host_slow_tier())
    torch.cuda.synchronize()
    assert ss.status() == tg.TG_OK
    _check(db, sp, lay)


def test_fp32_output_plan_equals_bf16_call():
    sp = synth.small(2)
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0)
    db.run()
    B = lay.kv_len.shape[0]
    shape = tg.make_shape(B, sp.Hq, sp.Hkv, sp.D, lay.num_pages)
    p32 = tg.tg_plan_create(shape, lay.kv_len, lay.group_of_head, lay.group_off, out_f32=True)
    o32 = torch.empty(db.out.shape, dtype=torch.float32, device="cuda")
    l32 = torch.empty_like(db.lse)
    tg.tg_ragged_paged_decode(p32, db.q, db.k, db.v, db.table, db.head_off, db.kv_len,
                              db.group_of_head, sp.scale, o32, l32)
    torch.cuda.synchronize()
    assert tg.tg_plan_status(p32) == tg.TG_OK
    assert torch.equal(o32.to(torch.bfloat16), db.out)
    assert torch.equal(l32, db.lse)


def test_pageable_host_tier_is_rejected():
    sp = synth.small(5)
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, min_splits=8, max_chunk_pages=16)
    ss = db.slow_stream(64, 2)
    with pytest.raises(ValueError):
        db.run_streamed(ss, tuple(t.cpu() for t in (db.k_q8, db.v_q8, db.k_scale, db.v_scale)))
