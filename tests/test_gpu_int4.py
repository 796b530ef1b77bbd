"""GPU parity of the INT4 slow tier: the quantiser's packed bytes and scales bit for bit against
the oracle's, and the tiered decode over an INT4 tier (HBM-resident and streamed from host
memory) against the fp64 oracle (out <= 2e-2, lse <= 1e-3) across plan shapes.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import non_uniform_paged_flash_b200 as tg
import oracle
import synth
from non_uniform_paged_flash_b200 import workload
from tests import _oracle_side as ors

pytestmark = pytest.mark.gpu


def _spec():
    return replace(synth.small(5), slow_bits=4)


def _check(db, sp, lay):
    ol = ors.layout(sp, 0)
    ors.assert_same_layout(lay, ol)
    ref_out, ref_lse = ors.reference(sp, ol, 0)
    out = db.out.float().cpu().numpy().reshape(-1, sp.D)
    lse = db.lse.cpu().numpy().reshape(-1)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin)
    e_o = np.abs(out - ref_out).max()
    e_l = np.abs(lse[fin] - ref_lse[fin]).max()
    assert e_o <= 2e-2, e_o
    assert e_l <= 1e-3, e_l


@pytest.mark.parametrize("D", [64, 128])
def test_quantize_int4_bit_exact(D):
    rng = np.random.default_rng(70 + D)
    x = synth.f64_to_bf16_bits(rng.normal(size=(777, D)) * rng.uniform(0.01, 30, (777, 1)))
    x[5] = 0                                               # amax = 0
    x[6] = synth.f64_to_bf16_bits(np.tile([3.5, 0.25, 1.25, -0.75], D // 4))  # ties
    src = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    packed = torch.empty((777, D // 2), dtype=torch.uint8, device="cuda")
    scale = torch.empty(777, dtype=torch.float32, device="cuda")
    tg.tg_quantize_int4(src, packed, scale)
    torch.cuda.synchronize()
    op, osc = oracle.quantize_int4(x)
    np.testing.assert_array_equal(packed.cpu().numpy(), op)
    np.testing.assert_array_equal(scale.cpu().numpy(), osc)


@pytest.mark.parametrize("kw", [dict(min_splits=8, max_chunk_pages=16),
                                dict(num_workers=1),
                                dict(num_workers=13, static_permille=200, dyn_chunk_pages=4),
                                dict(min_splits=64, max_chunk_pages=128, static_permille=900,
                                     dyn_chunk_pages=32, early_prologue=True)])
def test_int4_tier_matches_oracle(kw):
    sp = _spec()
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, **kw)
    assert db.k_q8.dtype == torch.uint8 and db.k_q8.shape[-1] == sp.D // 2
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK
    _check(db, sp, lay)


def test_int4_tier_streamed_from_host_matches_oracle():
    sp = _spec()
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, min_splits=8, max_chunk_pages=16)
    ss = db.slow_stream(9, 2, min_splits=4)
    db.run_streamed(ss, db.host_slow_tier())
    torch.cuda.synchronize()
    assert ss.status() == tg.TG_OK
    _check(db, sp, lay)


def test_int4_kv_bytes_are_about_half():
    sp = synth.small(5)
    lay = workload.layout(sp, 0)
    d8 = workload.to_device(sp, lay, 0)
    d4 = workload.to_device(replace(sp, slow_bits=4), lay, 0)
    b8, b4 = tg.tg_plan_get_info(d8.plan)["kv_bytes"], tg.tg_plan_get_info(d4.plan)["kv_bytes"]
    ns = int((lay.kv_len - np.minimum(lay.fast_len, lay.kv_len)).sum())
    assert b8 - b4 == ns * 2 * (sp.D // 2)
