"""GPU parity of the lean decode kernel (whole-head plans whose heads hold at most 64 pages: one
CTA per (sequence, KV head), plain 16-byte loads, fp32 softmax) against the fp64 oracle, at
every group size and head dimension, with empty heads, heads of exactly 64 pages and ragged
tails; its range checks; and its fp32 output form."""
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


def _is_lean(plan):
    info = tg.tg_plan_get_info(plan)
    return info["stages"] == 0 and info["block"] == 256 and info["n_merge"] == 0


def _check(db, sp, lay, layer=0):
    ol = ors.layout(sp, layer)
    ref_out, ref_lse = ors.reference(sp, ol, layer)
    out = db.out.float().cpu().numpy().reshape(-1, sp.D).astype(np.float64)
    lse = db.lse.cpu().numpy().reshape(-1).astype(np.float64)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin), "empty heads give lse = -inf"
    assert np.all(out[~fin] == 0.0), "empty heads give out = 0"
    assert np.abs(out - ref_out).max() <= OUT_TOL
    if fin.any():
        assert np.abs(lse[fin] - ref_lse[fin]).max() <= LSE_TOL
    return ref_out, ref_lse


@pytest.mark.parametrize("span", [(0, 1024), (0, 20)])
@pytest.mark.parametrize("early", [False, True])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
def test_lean_matches_oracle(G, D, early, span):
    # lengths drawn in [0, 1024] (several chunks, ragged tails, up to 64 pages) or [0, 20]
    # (empty heads, single tokens, one or two pages)
    sp = synth.Spec("lean sweep", "direct", B=5, Hq=3 * G, Hkv=3, D=D, len_lo=span[0],
                    len_hi=span[1], seed=0x7A4E4000 + 10 * G + D + span[1])
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, whole_heads=True, early_prologue=early)
    assert _is_lean(db.plan)
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK
    _check(db, sp, lay)
    a = db.out.clone(), db.lse.clone()
    db.run()
    torch.cuda.synchronize()
    assert torch.equal(a[0], db.out) and torch.equal(a[1], db.lse)   # deterministic


def test_lean_full_pages_and_64_page_heads():
    sp = synth.Spec("lean edges", "direct", B=3, Hq=8, Hkv=2, D=128, len_lo=1008, len_hi=1024,
                    seed=0x7A4E4100)
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, whole_heads=True)
    assert _is_lean(db.plan)
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK
    _check(db, sp, lay)


def test_longer_heads_keep_the_pipelined_kernel():
    sp = synth.Spec("not lean", "direct", B=2, Hq=8, Hkv=2, D=128, len_lo=1025, len_hi=2000,
                    seed=0x7A4E4200)
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, whole_heads=True)
    assert not _is_lean(db.plan)
    db.run()
    torch.cuda.synchronize()
    _check(db, sp, lay)


def test_lean_config1_is_one_launch_and_matches():
    sp = synth.preset(1)
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, **workload.timed_plan_options(1))
    assert _is_lean(db.plan)
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK
    _check(db, sp, lay)


def test_lean_bad_page_and_length_mismatch_are_reported():
    sp = synth.Spec("lean checks", "direct", B=4, Hq=8, Hkv=2, D=64, len_lo=40, len_hi=300,
                    seed=0x7A4E4300)
    lay = workload.layout(sp, 0)
    ol = ors.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, whole_heads=True)
    assert _is_lean(db.plan)
    ref_out, ref_lse = ors.reference(sp, ol, 0)
    G = sp.Hq // sp.Hkv
    bad = 3                                       # (b, h) = (1, 1)
    at = int(lay.head_off.reshape(-1)[bad])
    saved = db.table.clone()
    db.table[at] = lay.num_pages + 7              # outside the pool: skipped, never read
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_EBADPAGE
    keep = np.ones(sp.B * sp.Hq, bool)
    keep[bad * G:(bad + 1) * G] = False
    out = db.out.float().cpu().numpy().reshape(-1, sp.D)
    assert np.abs(out[keep] - ref_out[keep]).max() <= OUT_TOL
    db.table.copy_(saved)
    db.kv_len[0, 0] += 1                          # lengths that differ from the plan
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_EBADPAGE
    db.kv_len[0, 0] -= 1
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK
    _check(db, sp, lay)


def test_lean_fp32_output():
    sp = synth.Spec("lean f32", "direct", B=3, Hq=8, Hkv=2, D=128, len_lo=1, len_hi=500,
                    seed=0x7A4E4400)
    lay = workload.layout(sp, 0)
    ol = ors.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, whole_heads=True)
    shape = tg.make_shape(sp.B, sp.Hq, sp.Hkv, sp.D, lay.num_pages, 0, sp.page)
    plan = tg.tg_plan_create(shape, lay.kv_len, lay.group_of_head, lay.group_off,
                             whole_heads=True, out_f32=True)
    assert _is_lean(plan)
    out = torch.empty((sp.B, sp.Hq, sp.D), dtype=torch.float32, device="cuda")
    lse = torch.empty((sp.B, sp.Hq), dtype=torch.float32, device="cuda")
    tg.tg_ragged_paged_decode(plan, db.q, db.k, db.v, db.table, db.head_off, db.kv_len,
                              db.group_of_head, sp.scale, out, lse)
    torch.cuda.synchronize()
    assert tg.tg_plan_status(plan) == tg.TG_OK
    ref_out, ref_lse = ors.reference(sp, ol, 0)
    # fp32 scores, probabilities and output: far inside the bf16 tolerance
    assert np.abs(out.cpu().numpy().reshape(-1, sp.D) - ref_out).max() <= 1e-4
    assert np.abs(lse.cpu().numpy().reshape(-1) - ref_lse).max() <= 1e-4
