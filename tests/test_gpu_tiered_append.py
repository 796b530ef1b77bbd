"""GPU parity of the tier migration (fast window -> INT8 or INT4 tier) and of the tiered decode of a
capacity plan (made once for the reserved sizes, valid as the tiers grow) against the oracle:
slot choices, lengths and both tiers' pools bit for bit (the moved rows quantised by the pinned
quantiser), the decode within 2e-2 / 1e-3 at several points of the growth.
"""
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


def _dev(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=dt)).cuda()


def _bf(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("bits", [8, 4])
def test_tiered_append_and_capacity_decode(bits):
    sp = synth.small(5)                     # 2 sequences, 2100 tokens, 300 in the fast tier
    lay = workload.layout(sp, 0)
    ol = ors.layout(sp, 0)
    ors.assert_same_layout(lay, ol)
    B, Hkv = ol.kv_len.shape
    n0 = ol.kv_len.astype(np.int64)
    f0 = ol.fast_len.astype(np.int64)
    cap = int(f0.max())
    assert (f0 == cap).all() and (n0 % cap == 0).all()     # fast slot i holds position n - cap + i
    T = 40
    S = int((n0 - f0).max()) + T                           # reserved INT8 slots per head
    ps = -(-S // 16)
    Ps = B * Hkv * ps
    rng = np.random.default_rng(46)
    slow_table = rng.permutation(Ps).astype(np.int32)
    slow_off = (np.arange(B * Hkv, dtype=np.int64) * ps).reshape(B, Hkv)

    # INT8 tier contents: seeded bf16 rows quantised by the library / by the oracle
    ks_bits = synth.pool_bits(sp, "kslow", Ps)
    vs_bits = synth.pool_bits(sp, "vslow", Ps)
    quant = oracle.quantize_int4 if bits == 4 else oracle.quantize_int8
    kq_exp, ksc_exp = quant(ks_bits)        # INT4: packed bytes
    vq_exp, vsc_exp = quant(vs_bits)
    codes = oracle.unpack_int4 if bits == 4 else (lambda x: x)
    kq = torch.empty((Ps, 16, sp.D // 2 if bits == 4 else sp.D),
                     dtype=torch.uint8 if bits == 4 else torch.int8, device="cuda")
    vq = torch.empty_like(kq)
    ksc = torch.empty((Ps, 16), dtype=torch.float32, device="cuda")
    vsc = torch.empty_like(ksc)
    (tg.tg_quantize_int4 if bits == 4 else tg.tg_quantize_int8)(_bf(ks_bits), kq, ksc)
    (tg.tg_quantize_int4 if bits == 4 else tg.tg_quantize_int8)(_bf(vs_bits), vq, vsc)
    append = tg.tg_tiered_append_int4 if bits == 4 else tg.tg_tiered_append
    kf_exp = synth.pool_bits(sp, "k", ol.num_pages)
    vf_exp = synth.pool_bits(sp, "v", ol.num_pages)
    kf, vf = _bf(kf_exp), _bf(vf_exp)
    ftab, foff = _dev(lay.table, np.int32), _dev(lay.head_off, np.int64)
    stab, soff = _dev(slow_table, np.int32), _dev(slow_off, np.int64)
    kv_dev, fl_dev = _dev(n0, np.int32), _dev(f0, np.int32)
    fcap = _dev(np.full(B * Hkv, cap), np.int32)
    scap = _dev(np.full(B * Hkv, S), np.int32)
    moved = torch.empty(B * Hkv, dtype=torch.int32, device="cuda")
    slot = torch.empty(B * Hkv, dtype=torch.int32, device="cuda")
    shape = tg.make_shape(B, sp.Hq, sp.Hkv, sp.D, ol.num_pages, Ps)

    # one capacity plan for the whole growth
    plan = tg.tg_plan_create(shape, f0 + S, lay.group_of_head, lay.group_off, fast_len=f0,
                             slow_table_len=Ps, num_workers=23, min_splits=8,
                             max_chunk_pages=16, capacity=True, slow_bits=bits)
    q_bits = synth.q_bits(sp)
    q = _bf(q_bits)
    out = torch.empty((B, sp.Hq, sp.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, sp.Hq), dtype=torch.float32, device="cuda")
    n, f = n0.reshape(-1).copy(), f0.reshape(-1).copy()
    hoff = ol.head_off.reshape(-1)
    soff_h = slow_off.reshape(-1)

    def check_decode():
        tg.tg_tiered_decode(plan, q, kq, vq, ksc, vsc, stab, soff, kf, vf, ftab, foff, kv_dev,
                            fl_dev, sp.scale, out, lse)
        torch.cuda.synchronize()
        assert tg.tg_plan_status(plan) == tg.TG_OK
        ro, rl = oracle.tiered_decode(q_bits, codes(kq_exp), codes(vq_exp), ksc_exp, vsc_exp,
                                      slow_table,
                                      slow_off, kf_exp, vf_exp, ol.table, ol.head_off,
                                      n.reshape(B, Hkv).astype(np.int32),
                                      f.reshape(B, Hkv).astype(np.int32), sp.scale)
        o = out.float().cpu().numpy().reshape(-1, sp.D)
        lv = lse.cpu().numpy().reshape(-1)
        assert np.abs(o - ro).max() <= OUT_TOL
        assert np.abs(lv - rl).max() <= LSE_TOL

    check_decode()
    for step in range(T):
        kn, vn = synth.new_kv_bits(sp, step, "k"), synth.new_kv_bits(sp, step, "v")
        append(shape, _bf(kn), _bf(vn), kf, vf, ftab, foff, fcap, kq, vq, ksc, vsc,
               stab, soff, scap, kv_dev, fl_dev, moved, slot)
        want_fs, want_si = np.empty(B * Hkv, np.int32), np.empty(B * Hkv, np.int32)
        for bh in range(B * Hkv):
            fs, si = oracle.tier_step(int(n[bh]), int(f[bh]), cap, S)
            want_fs[bh], want_si[bh] = fs, si
            assert fs >= 0
            b, h = divmod(bh, Hkv)
            fpid = ol.table[hoff[bh] + fs // 16]
            if si >= 0:
                spid = slow_table[soff_h[bh] + si // 16]
                for src, q8, sc in ((kf_exp, kq_exp, ksc_exp), (vf_exp, vq_exp, vsc_exp)):
                    c, s_ = quant(src[fpid, fs % 16][None, :])
                    q8[spid, si % 16] = c[0]
                    sc[spid, si % 16] = s_[0]
            kf_exp[fpid, fs % 16] = kn[b, h]
            vf_exp[fpid, fs % 16] = vn[b, h]
            n[bh] += 1
            f[bh] = min(f[bh] + 1, cap)
        np.testing.assert_array_equal(slot.cpu().numpy(), want_fs, err_msg=f"step {step}")
        np.testing.assert_array_equal(moved.cpu().numpy(), want_si, err_msg=f"step {step}")
        if step == T // 2:
            check_decode()
    np.testing.assert_array_equal(kv_dev.cpu().numpy().reshape(-1), n)
    np.testing.assert_array_equal(fl_dev.cpu().numpy().reshape(-1), f)
    np.testing.assert_array_equal(_bits(kf), kf_exp)
    np.testing.assert_array_equal(_bits(vf), vf_exp)
    np.testing.assert_array_equal(kq.cpu().numpy(), kq_exp)
    np.testing.assert_array_equal(vq.cpu().numpy(), vq_exp)
    np.testing.assert_array_equal(ksc.cpu().numpy().view(np.uint32), ksc_exp.view(np.uint32))
    np.testing.assert_array_equal(vsc.cpu().numpy().view(np.uint32), vsc_exp.view(np.uint32))
    check_decode()


def test_tiered_append_fills_the_window_then_migrates():
    """A head that starts with every token fast fills its window first, then migrates."""
    sp = synth.Spec("tier fill", "tiered", B=1, Hq=8, Hkv=2, D=128, len_lo=20, len_hi=20,
                    fast_tokens=40, groups=1, seed=0x7A4E7000)
    lay = workload.layout(sp, 0)
    ol = ors.layout(sp, 0)
    B, Hkv = ol.kv_len.shape
    cap, S = 40, 64
    n = ol.kv_len.reshape(-1).astype(np.int64).copy()
    f = ol.fast_len.reshape(-1).astype(np.int64).copy()
    assert (n == f).all() and (f < cap).all()
    # the fast rows must hold cap slots: use a fresh fast tier of 3 pages per head
    pf = -(-cap // 16)
    Pf = B * Hkv * pf
    ftab = np.arange(Pf, dtype=np.int32)
    foff = (np.arange(B * Hkv, dtype=np.int64) * pf).reshape(B, Hkv)
    kf_exp = synth.pool_bits(sp, "k", Pf)
    vf_exp = synth.pool_bits(sp, "v", Pf)
    ps = -(-S // 16)
    Ps = B * Hkv * ps
    stab = np.arange(Ps, dtype=np.int32)[::-1].copy()
    soff = (np.arange(B * Hkv, dtype=np.int64) * ps).reshape(B, Hkv)
    kq_exp = np.zeros((Ps, 16, sp.D), np.int8)
    vq_exp = np.zeros_like(kq_exp)
    ksc_exp = np.zeros((Ps, 16), np.float32)
    vsc_exp = np.zeros_like(ksc_exp)
    kf, vf = _bf(kf_exp), _bf(vf_exp)
    kq, vq = _dev(kq_exp, np.int8), _dev(vq_exp, np.int8)
    ksc, vsc = _dev(ksc_exp, np.float32), _dev(vsc_exp, np.float32)
    shape = tg.make_shape(B, sp.Hq, sp.Hkv, sp.D, Pf, Ps)
    kv_dev, fl_dev = _dev(n, np.int32), _dev(f, np.int32)
    moved = torch.empty(B * Hkv, dtype=torch.int32, device="cuda")
    slot = torch.empty(B * Hkv, dtype=torch.int32, device="cuda")
    args = (_dev(ftab, np.int32), _dev(foff, np.int64), _dev(np.full(B * Hkv, cap), np.int32),
            kq, vq, ksc, vsc, _dev(stab, np.int32), _dev(soff, np.int64),
            _dev(np.full(B * Hkv, S), np.int32), kv_dev, fl_dev, moved, slot)
    for step in range(50):
        kn, vn = synth.new_kv_bits(sp, step, "k"), synth.new_kv_bits(sp, step, "v")
        tg.tg_tiered_append(shape, _bf(kn), _bf(vn), kf, vf, *args)
        for bh in range(B * Hkv):
            fs, si = oracle.tier_step(int(n[bh]), int(f[bh]), cap, S)
            b, h = divmod(bh, Hkv)
            fpid = ftab[foff.reshape(-1)[bh] + fs // 16]
            if si >= 0:
                spid = stab[soff.reshape(-1)[bh] + si // 16]
                for src, q8, sc in ((kf_exp, kq_exp, ksc_exp), (vf_exp, vq_exp, vsc_exp)):
                    c, s_ = oracle.quantize_int8(src[fpid, fs % 16][None, :])
                    q8[spid, si % 16], sc[spid, si % 16] = c[0], s_[0]
            kf_exp[fpid, fs % 16], vf_exp[fpid, fs % 16] = kn[b, h], vn[b, h]
            n[bh] += 1
            f[bh] = min(f[bh] + 1, cap)
        assert (moved.cpu().numpy() >= 0).tolist() == [bool(n[i] - 1 >= cap) for i in range(B * Hkv)]
    np.testing.assert_array_equal(_bits(kf), kf_exp)
    np.testing.assert_array_equal(kq.cpu().numpy(), kq_exp)
    np.testing.assert_array_equal(vsc.cpu().numpy().view(np.uint32), vsc_exp.view(np.uint32))
    np.testing.assert_array_equal(fl_dev.cpu().numpy().reshape(-1), f)


def test_tiered_append_rejects_states_outside_the_rules():
    shape = tg.make_shape(1, 4, 1, 128, 4, 4)
    z = lambda v, dt=np.int32: _dev(np.array(v), dt)
    kn = torch.zeros((1, 1, 128), dtype=torch.bfloat16, device="cuda")
    kf = torch.zeros((4, 16, 128), dtype=torch.bfloat16, device="cuda")
    kq = torch.zeros((4, 16, 128), dtype=torch.int8, device="cuda")
    sc = torch.zeros((4, 16), dtype=torch.float32, device="cuda")
    kv, fl = z([10]), z([2])                       # not full, yet older tokens exist
    moved, slot = z([7]), z([7])
    tg.tg_tiered_append(shape, kn, kn, kf, kf, z([0, 1]), z([0], np.int64), z([3]), kq, kq, sc, sc,
                        z([2, 3]), z([0], np.int64), z([32]), kv, fl, moved, slot)
    torch.cuda.synchronize()
    assert slot.item() == -1 and moved.item() == -1
    assert kv.item() == 10 and fl.item() == 2
