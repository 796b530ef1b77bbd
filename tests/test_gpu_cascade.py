"""GPU parity of the prefix-aware cascade (shared runs read once per step by dense tiles of query
rows, then merged with each head's private items) against the fp64 oracle: out within 2e-2,
lse within 1e-3, on the prefix workload (small: all rows; full size: sampled rows, in the
launch configuration the bench times) and on random prefix trees for every GQA group size and
both head dimensions.
"""
import numpy as np
import pytest
import torch

import non_uniform_paged_flash_b200 as tg
import oracle
import synth
from non_uniform_paged_flash_b200 import workload
from tests import _oracle_side as ors
from tests.test_cascade_plan import _random_tree_layout, check_cascade

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-2
LSE_TOL = 1e-3


def _compare(out, lse, ref_out, ref_lse, D, sel=None):
    o = out.float().cpu().numpy().reshape(-1, D).astype(np.float64)
    lv = lse.cpu().numpy().reshape(-1).astype(np.float64)
    if sel is not None:
        o, lv = o[sel], lv[sel]
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lv), fin)
    assert np.abs(o - ref_out).max() <= OUT_TOL, np.abs(o - ref_out).max()
    assert np.abs(lv[fin] - ref_lse[fin]).max() <= LSE_TOL, np.abs(lv[fin] - ref_lse[fin]).max()


@pytest.mark.parametrize("workers,min_readers", [(0, 2), (13, 2), (1, 3), (300, 5)])
def test_prefix_small_all_rows(workers, min_readers):
    sp = synth.small(4)
    lay = workload.layout(sp, 0)
    ol = ors.layout(sp, 0)
    ors.assert_same_layout(lay, ol)
    db = workload.to_device(sp, lay, 0, num_workers=workers, cascade=True,
                            min_readers=min_readers, static_permille=800, dyn_chunk_pages=2)
    assert tg.tg_plan_get_info(db.plan)["n_cascade"] > 0
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK
    ro, rl = ors.reference(sp, ol, 0)
    _compare(db.out, db.lse, ro, rl, sp.D)
    # repeated calls are bit-identical
    a = db.out.clone(), db.lse.clone()
    db.run()
    torch.cuda.synchronize()
    assert torch.equal(a[0], db.out) and torch.equal(a[1], db.lse)


def test_prefix_full_size_sampled_rows():
    sp = synth.preset(4)
    lay = workload.layout(sp, 0)
    ol = ors.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, cascade=True, static_permille=1000, early_prologue=True)
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK
    rng = np.random.default_rng(44)
    sel = np.sort(rng.choice(sp.B * sp.Hq, size=256, replace=False))
    ro, rl = ors.reference(sp, ol, 0, sel=sel)
    _compare(db.out, db.lse, ro, rl, sp.D, sel)


@pytest.mark.parametrize("G,D", [(1, 128), (2, 128), (4, 128), (8, 128), (4, 64), (8, 64)])
def test_random_prefix_trees(G, D):
    rng = np.random.default_rng(200 + 10 * G + D)
    B, Hkv = 70, 2
    table, head_off, kv, P = _random_tree_layout(rng, B, Hkv, n_roots=2, depth=3, fan=3)
    Hq = G * Hkv
    sp = synth.Spec("cascade trees", "direct", B=B, Hq=Hq, Hkv=Hkv, D=D, len_lo=1, len_hi=2,
                    seed=0x7A4E6000 + 10 * G + D)
    k = synth.pool_bits(sp, "k", P)
    v = synth.pool_bits(sp, "v", P)
    q = synth.q_bits(sp)
    scale = 1.0 / np.sqrt(D)
    shape = tg.make_shape(B, Hq, Hkv, D, P)
    goh = np.zeros(Hkv, np.int32)
    goff = np.array([0, table.size], np.int64)
    plan = tg.tg_plan_create_cascade(shape, kv, goh, goff, table, head_off, num_workers=37,
                                     static_permille=700, dyn_chunk_pages=3)
    check_cascade(plan, B, Hq, Hkv, kv, table, head_off)
    assert tg.tg_plan_get_info(plan)["n_cascade"] > 0
    bf = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()
    it = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dtype=dt)).cuda()
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    tg.tg_ragged_paged_decode(plan, bf(q), bf(k), bf(v), it(table, np.int32), it(head_off, np.int64),
                              it(kv, np.int32), it(goh, np.int32), float(scale), out, lse)
    torch.cuda.synchronize()
    assert tg.tg_plan_status(plan) == tg.TG_OK
    ro, rl = oracle.decode(q, k, v, table, head_off, kv, scale)
    _compare(out, lse, ro, rl, D)


def test_cascade_bad_page_is_reported():
    """A shared page id outside the pool is skipped by the cascade and reported."""
    sp = synth.small(4)
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, cascade=True)
    db.table[int(lay.head_off.reshape(-1)[0])] = lay.num_pages + 7   # page 0 of (0, 0): shared
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_EBADPAGE
