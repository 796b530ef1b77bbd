"""GPU parity of the SplitZip codec against the oracle: every stream (codebook, sign/mantissa
bytes, packed codes, escape count, positions, exponents) bit for bit, and lossless decoding of
both the GPU's and the oracle's streams, over tile-edge sizes, escape-heavy data and a full
K/V pool.
"""
import numpy as np
import pytest
import torch

import non_uniform_paged_flash_b200 as tg
import oracle
import synth

pytestmark = pytest.mark.gpu


def _dev(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=dt)).cuda()


def _encode(x_bits, cap=None):
    n = x_bits.size
    cap = n if cap is None else cap
    src = _dev(x_bits.view(np.int16) if n else np.zeros(8, np.int16), np.int16)
    cb = torch.empty(16, dtype=torch.uint8, device="cuda")
    sm = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    codes = torch.empty(max((n + 1) // 2, 8), dtype=torch.uint8, device="cuda")
    pos = torch.full((max(cap, 1),), -1, dtype=torch.int64, device="cuda")
    exp = torch.zeros(max(cap, 1), dtype=torch.uint8, device="cuda")
    n_esc = torch.zeros(1, dtype=torch.int64, device="cuda")
    ws = torch.empty(tg.tg_splitzip_workspace_bytes(n), dtype=torch.uint8, device="cuda")
    tg.tg_splitzip_encode(n, src, cb, sm, codes, pos[:cap] if cap else None,
                          exp[:cap] if cap else None, n_esc, ws)
    torch.cuda.synchronize()
    return cb, sm, codes, pos, exp, n_esc


def _kinds(rng, n):
    normal = synth.f64_to_bf16_bits(rng.normal(size=n) * 2)
    anybits = rng.integers(0, 1 << 16, n).astype(np.uint16)
    special = np.array([0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC0, 0x0001, 0x807F], np.uint16)
    anybits[rng.integers(0, max(n, 1), min(n, 30))] = rng.choice(special, min(n, 30))
    heavy = synth.f64_to_bf16_bits(rng.standard_cauchy(n) * 1e3)     # many rare exponents
    return {"normal": normal, "anybits": anybits, "heavy": heavy}


@pytest.mark.parametrize("n", [0, 1, 7, 15, 16, 4095, 4096, 4097, 100003])
def test_encode_matches_oracle_and_round_trips(n):
    rng = np.random.default_rng(50 + n)
    for kind, x in _kinds(rng, n).items():
        cb, sm, codes, pos, exp, n_esc = _encode(x)
        ocb, osm, ocodes, opos, oexp = oracle.splitzip_encode(x)
        k = int(n_esc.item())
        assert k == opos.size, kind
        np.testing.assert_array_equal(cb.cpu().numpy(), ocb, err_msg=kind)
        np.testing.assert_array_equal(sm.cpu().numpy()[:n], osm, err_msg=kind)
        np.testing.assert_array_equal(codes.cpu().numpy()[:(n + 1) // 2], ocodes, err_msg=kind)
        np.testing.assert_array_equal(pos.cpu().numpy()[:k], opos, err_msg=kind)
        np.testing.assert_array_equal(exp.cpu().numpy()[:k], oexp, err_msg=kind)
        if n == 0:
            continue
        for streams in ((cb, sm, codes, pos[:max(k, 1)], exp[:max(k, 1)], n_esc),
                        (_dev(ocb, np.uint8), _dev(np.resize(osm, max(n, 16)), np.uint8),
                         _dev(np.resize(ocodes, max((n + 1) // 2, 8)), np.uint8),
                         _dev(opos if k else np.zeros(1), np.int64),
                         _dev(oexp if k else np.zeros(1), np.uint8), _dev([k], np.int64))):
            dst = torch.empty(n + 8, dtype=torch.int16, device="cuda")
            tg.tg_splitzip_decode(n, *streams[:3], streams[3], streams[4], streams[5], dst)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(dst.cpu().numpy()[:n].view(np.uint16), x, err_msg=kind)


def test_escape_capacity_overflow_reports_the_true_count():
    rng = np.random.default_rng(51)
    x = _kinds(rng, 20000)["anybits"]
    opos = oracle.splitzip_encode(x)[3]
    cap = opos.size // 3
    cb, sm, codes, pos, exp, n_esc = _encode(x, cap=cap)
    assert int(n_esc.item()) == opos.size
    np.testing.assert_array_equal(pos.cpu().numpy()[:cap], opos[:cap])


def test_full_pool_round_trip():
    """The K pool of the GQA decode workload (config 2, 0.33 GB of bf16)."""
    sp = synth.preset(2)
    from non_uniform_paged_flash_b200 import workload
    lay = workload.layout(sp, 0)
    k = workload._pool_to_device(sp, "k", lay.num_pages, "cuda")
    n = k.numel()
    flat = k.view(torch.int16).reshape(-1)
    cb = torch.empty(16, dtype=torch.uint8, device="cuda")
    sm = torch.empty(n, dtype=torch.uint8, device="cuda")
    codes = torch.empty((n + 1) // 2, dtype=torch.uint8, device="cuda")
    cap = n // 20
    pos = torch.empty(cap, dtype=torch.int64, device="cuda")
    exp = torch.empty(cap, dtype=torch.uint8, device="cuda")
    n_esc = torch.zeros(1, dtype=torch.int64, device="cuda")
    ws = torch.empty(tg.tg_splitzip_workspace_bytes(n), dtype=torch.uint8, device="cuda")
    tg.tg_splitzip_encode(n, flat, cb, sm, codes, pos, exp, n_esc, ws)
    dst = torch.empty_like(flat)
    tg.tg_splitzip_decode(n, cb, sm, codes, pos, exp, n_esc, dst)
    torch.cuda.synchronize()
    assert int(n_esc.item()) <= cap
    assert torch.equal(dst, flat)
    # codebook and escape count against the oracle on the same values
    bits = flat.cpu().numpy().view(np.uint16)
    ocb, _, _, opos, _ = oracle.splitzip_encode(bits)
    np.testing.assert_array_equal(cb.cpu().numpy(), ocb)
    assert int(n_esc.item()) == opos.size
