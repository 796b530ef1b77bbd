"""The decode entry point that allocates no device memory, for callers that cannot allocate
after start-up (an engine that reserves the whole device for its KV pool, a plug-in whose host
framework owns every device allocation). It must give the oracle's results, and those of the
plan-based entry point, call after call, with its scratch in the library's fixed device array;
its error word must report a wait that ran out.

Kept in a file of its own, collected last: if it fails, every other test has already run."""
import numpy as np
import pytest
import torch

import non_uniform_paged_flash_b200 as tg
import synth
from non_uniform_paged_flash_b200 import workload
from tests import _oracle_side as ors

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-2
LSE_TOL = 1e-3


def _host_plan(sp, lay, **kw):
    shape = tg.make_shape(sp.B, sp.Hq, sp.Hkv, sp.D, lay.num_pages, 0, sp.page)
    return tg.tg_plan_create(shape, lay.kv_len, lay.group_of_head, lay.group_off,
                             host_only=True, **kw)


def _noalloc(hp, db, sp):
    out = torch.full_like(db.out, float("nan"))
    lse = torch.full_like(db.lse, float("nan"))
    tg.tg_ragged_paged_decode_noalloc(hp, db.q, db.k, db.v, db.table, db.head_off,
                                      db.kv_len, db.group_of_head, sp.scale, out, lse)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("cfg,kw", [(2, dict(num_workers=64, static_permille=800)),
                                    (1, dict(num_workers=8, static_permille=1000))])
def test_no_alloc_matches_oracle_and_plan_entry_point_twice(cfg, kw):
    sp = synth.small(cfg) if cfg != 1 else synth.preset(1)
    lay = workload.layout(sp, 0)
    ol = ors.layout(sp, 0)
    ors.assert_same_layout(lay, ol)
    ref_out, ref_lse = ors.reference(sp, ol, 0)            # fp64 oracle
    fin = np.isfinite(ref_lse)
    db = workload.to_device(sp, lay, 0, **kw)
    db.run()
    torch.cuda.synchronize()
    plan_out, plan_lse = db.out.float().clone(), db.lse.clone()
    hp = _host_plan(sp, lay, **kw)
    info = tg.tg_plan_get_info(hp)
    assert info["device_bytes"] == 0                       # the plan holds no device memory
    if cfg == 2:
        assert info["n_partials"] > 0 and info["n_dynamic"] > 0   # scratch is really used
    for _ in range(2):                                     # the scratch keeps the last call
        out, lse = _noalloc(hp, db, sp)
        assert tg.tg_ragged_paged_decode_noalloc_status() == tg.TG_OK
        o = out.float().cpu().numpy().reshape(-1, sp.D)
        l = lse.cpu().numpy().reshape(-1)
        assert np.array_equal(np.isfinite(l), fin)
        assert np.abs(o - ref_out).max() <= OUT_TOL
        assert np.abs(l[fin] - ref_lse[fin]).max() <= LSE_TOL
        f = torch.isfinite(plan_lse)
        assert (out.float() - plan_out).abs().max().item() <= OUT_TOL
        assert (lse[f] - plan_lse[f]).abs().max().item() <= LSE_TOL


def test_no_alloc_reports_a_wait_that_ran_out():
    """A page the producer never signals (the plan's test hook; a flag nothing sets) makes the
    consumer's bounded wait run out: the call's kernels return, the status call reports
    TG_ETIMEOUT and clears the word, and the next call is clean and correct."""
    sp = synth.small(2)
    lay = workload.layout(sp, 0)
    ol = ors.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, num_workers=16)
    hp = _host_plan(sp, lay, num_workers=16, wait_limit_us=20000, test_withhold_page=2)
    _noalloc(hp, db, sp)
    assert tg.tg_ragged_paged_decode_noalloc_status() == tg.TG_ETIMEOUT
    assert tg.tg_ragged_paged_decode_noalloc_status() == tg.TG_OK     # read and cleared
    hp = _host_plan(sp, lay, num_workers=16, wait_limit_us=20000)
    out, lse = _noalloc(hp, db, sp)
    assert tg.tg_ragged_paged_decode_noalloc_status() == tg.TG_OK
    ref_out, ref_lse = ors.reference(sp, ol, 0)
    fin = np.isfinite(ref_lse)
    assert np.abs(out.float().cpu().numpy().reshape(-1, sp.D) - ref_out).max() <= OUT_TOL
    assert np.abs(lse.cpu().numpy().reshape(-1)[fin] - ref_lse[fin]).max() <= LSE_TOL


def test_no_alloc_refuses_a_plan_of_another_device():
    sp = synth.small(2)
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, num_workers=16)
    other = torch.cuda.current_device() + 1                # never touched: refused on the host
    hp = _host_plan(sp, lay, num_workers=16, device=other)
    with pytest.raises(tg.TGError) as e:
        tg.tg_ragged_paged_decode_noalloc(hp, db.q, db.k, db.v, db.table, db.head_off,
                                          db.kv_len, db.group_of_head, sp.scale, db.out, db.lse)
    assert e.value.status == tg.TG_EINVAL


def test_no_alloc_rejects_plans_beyond_its_scratch():
    sp = synth.preset(4)
    lay = workload.layout(sp, 0)
    hp = _host_plan(sp, lay, num_workers=60000, static_permille=1000)
    assert tg.tg_plan_get_info(hp)["n_partials"] * 4 * 129 * 4 > 16 << 20
    q = torch.zeros((sp.B, sp.Hq, sp.D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty((sp.B, sp.Hq), dtype=torch.float32, device="cuda")
    dummy = torch.zeros(16, dtype=torch.int64, device="cuda")
    with pytest.raises(tg.TGError) as e:
        tg.tg_ragged_paged_decode_noalloc(hp, q, q, q, dummy, dummy, dummy, dummy, sp.scale,
                                          out, lse)
    assert e.value.status == tg.TG_ENOMEM
