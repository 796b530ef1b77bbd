"""The decode entry point that allocates no device memory, for callers that cannot allocate
after start-up (an engine that reserves the whole device for its KV pool, a plug-in whose host
framework owns every device allocation). It must give the results of the plan-based entry
point, call after call, with its scratch in the library's fixed device array.

Kept in a file of its own, collected last: if it fails, every other test has already run."""
import pytest
import torch

import non_uniform_paged_flash_b200 as tg
import synth
from non_uniform_paged_flash_b200 import workload

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-2
LSE_TOL = 1e-3


def _host_plan(sp, lay, **kw):
    shape = tg.make_shape(sp.B, sp.Hq, sp.Hkv, sp.D, lay.num_pages, 0, sp.page)
    return tg.tg_plan_create(shape, lay.kv_len, lay.group_of_head, lay.group_off,
                             host_only=True, **kw)


@pytest.mark.parametrize("cfg,kw", [(2, dict(num_workers=64, static_permille=800)),
                                    (1, dict(num_workers=8, static_permille=1000))])
def test_no_alloc_matches_plan_entry_point_twice(cfg, kw):
    sp = synth.small(cfg) if cfg != 1 else synth.preset(1)
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, **kw)
    db.run()
    torch.cuda.synchronize()
    ref_out, ref_lse = db.out.float().clone(), db.lse.clone()
    hp = _host_plan(sp, lay, **kw)
    info = tg.tg_plan_get_info(hp)
    assert info["device_bytes"] == 0                       # the plan holds no device memory
    if cfg == 2:
        assert info["n_partials"] > 0 and info["n_dynamic"] > 0   # scratch is really used
    for _ in range(2):                                     # the scratch keeps the last call
        out = torch.full_like(db.out, float("nan"))
        lse = torch.full_like(db.lse, float("nan"))
        tg.tg_ragged_paged_decode_noalloc(hp, db.q, db.k, db.v, db.table, db.head_off,
                                          db.kv_len, db.group_of_head, sp.scale, out, lse)
        torch.cuda.synchronize()
        fin = torch.isfinite(ref_lse)
        assert torch.equal(torch.isfinite(lse), fin)
        assert (out.float() - ref_out).abs().max().item() <= OUT_TOL
        assert (lse[fin] - ref_lse[fin]).abs().max().item() <= LSE_TOL


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
