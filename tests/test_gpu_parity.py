"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Tolerances: max |out - oracle| <= 2e-2 on the bf16 outputs and max |lse - oracle| <= 1e-3 on
the fp32 log-sum-exp (the target this library is held to). Layouts are compared bit for bit
with the oracle's own derivation before any numerics. INT8 codes and scales must be bit-exact.
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

OUT_TOL = 2e-2
LSE_TOL = 1e-3


def _compare(db, ref_out, ref_lse, sel=None):
    out = db.out.float().cpu().numpy().reshape(-1, db.spec.D).astype(np.float64)
    lse = db.lse.cpu().numpy().reshape(-1).astype(np.float64)
    if sel is not None:
        out, lse = out[sel], lse[sel]
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin), "empty rows must give lse = -inf"
    assert np.all(out[~fin] == 0.0), "empty rows must give out = 0"
    err_o = np.abs(out - ref_out).max() if out.size else 0.0
    err_l = np.abs(lse[fin] - ref_lse[fin]).max() if fin.any() else 0.0
    assert err_o <= OUT_TOL, f"max |out - oracle| = {err_o}"
    assert err_l <= LSE_TOL, f"max |lse - oracle| = {err_l}"
    return err_o, err_l


def _run(sp, layer=0, sel=None, **plan_kw):
    lay = workload.layout(sp, layer)
    ol = ors.layout(sp, layer)
    ors.assert_same_layout(lay, ol)
    db = workload.to_device(sp, lay, layer, **plan_kw)
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK
    ref_out, ref_lse = ors.reference(sp, ol, layer, sel=sel)
    return db, _compare(db, ref_out, ref_lse, sel)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("workers", [0, 1, 13])
@pytest.mark.parametrize("static_permille", [1000, 800, 200])
def test_small_configs_match_oracle(cfg, workers, static_permille):
    sp = synth.small(cfg)
    kw = dict(num_workers=workers, static_permille=static_permille, dyn_chunk_pages=4)
    if cfg == 5:
        kw.update(min_splits=8, max_chunk_pages=16)
    for layer in range(min(sp.layers, 2)):
        _run(sp, layer, **kw)


@pytest.mark.parametrize("cfg", [1, 2])
@pytest.mark.parametrize("workers", [0, 3])
def test_whole_head_plans_match_oracle(cfg, workers):
    """whole_heads plans: one item per head, no merge kernel."""
    sp = synth.small(cfg)
    db, _ = _run(sp, num_workers=workers, whole_heads=True)
    assert tg.tg_plan_get_info(db.plan)["n_merge"] == 0


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
def test_gqa_and_head_dims(G, D):
    sp = synth.Spec("gqa sweep", "direct", B=3, Hq=2 * G, Hkv=2, D=D, len_lo=1, len_hi=700,
                    seed=0x7A4E1000 + 10 * G + D)
    _run(sp, num_workers=37)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("workers", [0, 37])
def test_tiered_gqa_sweep(G, bits, workers):
    """The tiered kernel at every group size it accepts (G = 8 runs a shallower ring: its
    stages hold 8 query rows), INT8 and INT4 slow tiers, ragged tail pages in both tiers
    (1300 slow = 81 pages + 4 tokens, 200 fast = 12 pages + 8 tokens), heads split into
    several items and merged."""
    sp = synth.Spec("tiered gqa sweep", "tiered", B=2, Hq=2 * G, Hkv=2, D=128, len_lo=1500,
                    len_hi=1500, fast_tokens=200, seed=0x7A4E1100 + 10 * G + bits,
                    slow_bits=bits)
    db, _ = _run(sp, num_workers=workers, min_splits=4, max_chunk_pages=16)
    assert tg.tg_plan_get_info(db.plan)["n_merge"] > 0


def test_empty_and_single_token_heads():
    sp = synth.Spec("edges", "direct", B=4, Hq=8, Hkv=4, D=128, len_lo=0, len_hi=2,
                    seed=0x7A4E2000)
    db, _ = _run(sp, num_workers=5)
    kv = db.lay.kv_len
    assert (kv == 0).any() and (kv == 1).any()
    # one retained token: out equals that token's V row exactly (bf16 -> bf16)
    v = synth.pool_bits(sp, "v", db.lay.num_pages)
    out = db.out.view(torch.int16).cpu().numpy().view(np.uint16)
    G = sp.Hq // sp.Hkv
    for b in range(sp.B):
        for h in range(sp.Hkv):
            if kv[b, h] == 1:
                pid = db.lay.table[db.lay.head_off[b, h]]
                for n in range(G):
                    np.testing.assert_array_equal(out[b, h * G + n], v[pid, 0])


def test_split_heads_every_partition_size():
    """Many workers over few heads: every head is cut into many items and merged."""
    sp = synth.Spec("splits", "direct", B=2, Hq=8, Hkv=2, D=128, len_lo=500, len_hi=3000,
                    seed=0x7A4E3000)
    for workers in (2, 3, 64, 400):
        db, _ = _run(sp, num_workers=workers)
        info = tg.tg_plan_get_info(db.plan)
        if workers >= 64:
            assert info["n_partials"] > 0


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("workers, lo, hi", [(8, 2, 8), (48, 9, 32), (400, 33, 10**6)])
def test_merge_by_parts_per_head(D, workers, lo, hi):
    """Each merge kernel, chosen by the most parts a head of the plan has (up to 8: a warp per
    row, parts 4 at a time; 9 to 32: a warp per row, a lane per part; more: a CTA per row),
    at both head dimensions, against the oracle. A head's parts are the workers its pages land
    on (at most one worker per 8 pages of the batch)."""
    sp = synth.Spec("merge", "direct", B=2, Hq=8, Hkv=2, D=D, len_lo=2000, len_hi=9000,
                    seed=0x7A4E3100 + D)
    db, _ = _run(sp, num_workers=workers, static_permille=1000)
    items = tg.tg_plan_items(db.plan)
    mi = items[:, 7]
    parts = np.bincount(mi[mi >= 0])
    assert lo <= parts.max() <= hi, parts.max()


def test_deterministic_repeat():
    """Dynamic items land on different workers from call to call; the merge order (split
    order) keeps the results bit-identical."""
    sp = synth.small(2)
    db, _ = _run(sp, static_permille=300, dyn_chunk_pages=2)
    a = db.out.clone(), db.lse.clone()
    for _ in range(3):
        db.run()
    torch.cuda.synchronize()
    assert torch.equal(a[0], db.out) and torch.equal(a[1], db.lse)


def test_quantizer_bit_exact():
    rng = np.random.default_rng(30)
    x = rng.normal(size=(4096, 128)) * rng.choice([1e-3, 1.0, 300.0], size=(4096, 1))
    x[0] = 0.0
    x[1, :] = 0.0
    x[1, 5] = -2.5
    bits = synth.f64_to_bf16_bits(x)
    gold = [[1.984375, 1.0, -0.5, 0.0078125, 0.0234375, 0.0390625, -0.0546875, -1.984375]]
    bits[2, :8] = synth.f64_to_bf16_bits(np.array(gold[0]))
    bits[2, 8:] = 0
    for D in (128, 64):
        b = np.ascontiguousarray(bits[:, :D])
        src = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda()
        codes = torch.empty((b.shape[0], D), dtype=torch.int8, device="cuda")
        scale = torch.empty(b.shape[0], dtype=torch.float32, device="cuda")
        tg.tg_quantize_int8(src, codes, scale)
        oc, os_ = oracle.quantize_int8(b)
        np.testing.assert_array_equal(codes.cpu().numpy(), oc)
        np.testing.assert_array_equal(scale.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    np.testing.assert_array_equal(oc[2, :8], [127, 64, -32, 0, 2, 2, -4, -127])


def test_lse_merge_entry_point():
    rng = np.random.default_rng(31)
    rows, D = 50, 128
    counts = rng.integers(0, 6, rows)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    S = int(off[-1])
    po = rng.normal(size=(S, D)).astype(np.float32)
    pl = (rng.normal(size=S) * 5).astype(np.float32)
    pl[rng.random(S) < 0.1] = -np.inf
    out = torch.empty((rows, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(rows, dtype=torch.float32, device="cuda")
    tg.tg_lse_merge(torch.from_numpy(off).cuda(), torch.from_numpy(po).cuda(),
                    torch.from_numpy(pl).cuda(), out, lse)
    torch.cuda.synchronize()
    Smax = max(1, int(counts.max()))
    PO = np.zeros((Smax, rows, D))
    PL = np.full((Smax, rows), -np.inf)
    for r in range(rows):
        for j in range(counts[r]):
            PO[j, r] = po[off[r] + j]
            PL[j, r] = pl[off[r] + j]
    ro, rl = oracle.lse_merge(PO, PL)
    o = out.float().cpu().numpy()
    l = lse.cpu().numpy()
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(l), fin)
    assert np.abs(o - ro).max() <= OUT_TOL
    assert np.abs(l[fin] - rl[fin]).max() <= LSE_TOL


def test_bad_page_id_is_reported_not_read():
    """A page id outside the pool is skipped and reported (TG_EBADPAGE); heads that do not
    read it are unaffected. The kernel checks the id before issuing the copy."""
    sp = synth.small(2)
    lay = workload.layout(sp, 0)
    ol = ors.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, num_workers=16)
    bad_row = 3                                    # (b, h) = (0, 3)
    bad_at = int(lay.head_off.reshape(-1)[bad_row])
    tbl = db.table.clone()
    db.table[bad_at] = lay.num_pages + 12345
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_EBADPAGE
    ref_out, ref_lse = ors.reference(sp, ol, 0)
    G = sp.Hq // sp.Hkv
    keep = np.ones(sp.B * sp.Hq, bool)
    keep[bad_row * G:(bad_row + 1) * G] = False    # rows of b = 0, h = 3
    out = db.out.float().cpu().numpy().reshape(-1, sp.D)
    lse = db.lse.cpu().numpy().reshape(-1)
    assert np.abs(out[keep] - ref_out[keep]).max() <= OUT_TOL
    assert np.abs(lse[keep] - ref_lse[keep]).max() <= LSE_TOL
    db.table.copy_(tbl)                            # restored table: clean again
    db.run()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK


def test_length_mismatch_with_plan_is_reported():
    sp = synth.small(1)
    db = workload.admit(sp)
    db.kv_len[0, 0] += 1
    db.run()
    assert tg.tg_plan_status(db.plan) == tg.TG_EBADPAGE


def test_bounded_wait_runs_out_and_context_survives():
    """A page that is never signalled (a flag nothing sets) makes the consumer's bounded wait
    run out: the kernel drains what it issued, returns, and the call reports TG_ETIMEOUT; the
    context stays usable and a normal plan afterwards gives correct results."""
    sp = synth.small(2)
    lay = workload.layout(sp, 0)
    ol = ors.layout(sp, 0)
    for withhold in (1, 3):
        db = workload.to_device(sp, lay, 0, num_workers=16, wait_limit_us=20000,
                                test_withhold_page=withhold)
        db.run()
        torch.cuda.synchronize()
        assert tg.tg_plan_status(db.plan) == tg.TG_ETIMEOUT
        del db
    db = workload.to_device(sp, lay, 0, num_workers=16, wait_limit_us=20000)
    db.run()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK
    ref_out, ref_lse = ors.reference(sp, ol, 0)
    _compare(db, ref_out, ref_lse)


def test_argument_validation():
    sp = synth.small(1)
    db = workload.admit(sp)
    big = torch.empty(db.out.numel() + 8, dtype=db.out.dtype, device=db.out.device)
    with pytest.raises(tg.TGError) as e:
        tg.tg_ragged_paged_decode(db.plan, db.q, db.k, db.v, db.table, db.head_off, db.kv_len,
                                  db.group_of_head, sp.scale, big[1:1 + db.out.numel()], db.lse)
    assert e.value.status == tg.TG_EINVAL          # misaligned output (the C ABI's check)
    with pytest.raises(ValueError):                 # too small (the binding's check)
        tg.tg_ragged_paged_decode(db.plan, db.q, db.k, db.v, db.table, db.head_off, db.kv_len,
                                  db.group_of_head, sp.scale, db.out.view(-1)[1:], db.lse)
    with pytest.raises(tg.TGError):
        tg.tg_tiered_decode(db.plan, db.q, None, None, None, None, None, None, db.k, db.v,
                            db.table, db.head_off, db.kv_len, db.kv_len, sp.scale, db.out, db.lse)


# ---------------------------------------------------------------------------------------
# Full sizes, in the launch configuration the bench times (default plan options).
# ---------------------------------------------------------------------------------------

def test_full_config1_all_rows():
    _run(synth.preset(1), **workload.timed_plan_options(1))


def test_full_config2_all_rows():
    _run(synth.preset(2), **workload.timed_plan_options(2))


def test_full_config2_default_plan_all_rows():
    _run(synth.preset(2))


def test_full_config3_all_rows_two_layers():
    """Every query row of two layers of the serving step (8192 rows each), in the plan options
    the bench times; the layers share the bench's one pool upload."""
    sp = synth.preset(3)
    for layer in (0, 17):
        _run(sp, layer, **workload.timed_plan_options(3))


def test_full_config4_all_rows():
    """The prefix-cascade plan the bench times (tcgen05 cascade + split-K items + merge), every
    one of the 16384 query rows."""
    sp = synth.preset(4)
    db, _ = _run(sp, **workload.timed_plan_options(4))
    assert tg.tg_plan_get_info(db.plan)["n_cascade"] > 0


def test_full_config5_all_rows():
    sp = synth.preset(5)
    _run(sp, **workload.timed_plan_options(5))


def test_full_config5_int4_all_rows():
    sp = replace(synth.preset(5), slow_bits=4)
    _run(sp, **workload.timed_plan_options(5))


@pytest.mark.parametrize("bits", [8, 4])
def test_full_config5_host_streamed_all_rows(bits):
    """The slow tier streamed from pinned host memory in 8192-page blocks through a ring of 3
    (the bench's ttkv-host configuration), every row against the oracle."""
    sp = replace(synth.preset(5), slow_bits=bits)
    lay = workload.layout(sp, 0)
    kw = {k: v for k, v in workload.timed_plan_options(5).items() if k != "early_prologue"}
    db = workload.to_device(sp, lay, 0, **kw)
    ss = db.slow_stream(8192, 3, **kw)
    db.run_streamed(ss, db.host_slow_tier())
    torch.cuda.synchronize()
    assert ss.status() == tg.TG_OK
    ol = ors.layout(sp, 0)
    ref_out, ref_lse = ors.reference(sp, ol, 0)
    _compare(db, ref_out, ref_lse)
