"""Pins for the CPU oracle: each oracle function is checked against something other than
itself — hand-worked values tied to the source pages (tests/golden/), closed forms,
textbook/library routines, invariants, and brute force on tiny inputs. Chosen so that a
dropped term, a wrong sign or index, or a transposed operand fails at least one of them.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests._paged import bf16, flat_table, scatter_rows, widen

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------------------
# Host-side steps: hand-worked examples from tests/golden.
# ---------------------------------------------------------------------------------------

def test_retained_lengths_golden():
    g = gold("retained_lengths.json")["cases"]
    L = np.array([c["L"] for c in g], np.int32)
    r = np.array([c["ratio_ppm"] for c in g], np.int32)
    exp = np.array([c["kv_len"] for c in g], np.int32)
    np.testing.assert_array_equal(oracle.retained_lengths(L, r), exp)


def test_retained_lengths_invariants():
    rng = np.random.default_rng(0)
    L = rng.integers(1, 200_000, 5000).astype(np.int32)
    r = rng.integers(0, 1_000_001, 5000).astype(np.int32)
    kv = oracle.retained_lengths(L, r)
    assert (kv >= 1).all() and (kv <= L).all()
    # |kv - ratio*L| <= 1/2 wherever the clamps are inactive (closed form of rounding)
    exact = r.astype(np.float64) * L / 1e6
    free = (exact >= 0.5) & (exact <= L - 0.5)
    assert (np.abs(kv[free] - exact[free]) <= 0.5 + 1e-9).all()
    # monotone in the ratio
    kv2 = oracle.retained_lengths(L, np.minimum(r + 1000, 1_000_000).astype(np.int32))
    assert (kv2 >= kv).all()


def test_budget_groups_golden():
    for c in gold("budget_groups.json")["cases"]:
        np.testing.assert_array_equal(oracle.budget_groups(c["budget_ppm"], c["G"]), c["group"])


def test_budget_groups_invariants():
    rng = np.random.default_rng(1)
    for n, G in [(8, 4), (256, 8), (7, 3), (32, 32)]:
        b = rng.integers(0, 10**6, n).astype(np.int32)
        g = oracle.budget_groups(b, G)
        counts = np.bincount(g, minlength=G)
        assert counts.max() - counts.min() <= 1          # equal-count quantiles
        # every head in a lower group has a budget <= every head in a higher group
        for a in range(G - 1):
            if counts[a] and counts[a + 1]:
                assert b[g == a].max() <= b[g == a + 1].min()


def test_reservation_layout_golden():
    for c in gold("reservation_layout.json")["cases"]:
        ids, cnt, segp = oracle.reservation_layout(
            c["num_pages"], c["free_order"], c["page"], np.array(c["kv_len"]),
            c["seg_tokens"], None if c["chain"] is None else np.array(c["chain"]))
        np.testing.assert_array_equal(ids, c["page_ids"])
        np.testing.assert_array_equal(cnt, c["head_count"])
        np.testing.assert_array_equal(segp, c["seg_pages"])


def test_reservation_layout_invariants():
    rng = np.random.default_rng(2)
    B, H, page = 9, 4, 16
    kv = rng.integers(0, 300, (B, H)).astype(np.int32)
    need = int(((kv + page - 1) // page).sum())
    order = rng.permutation(need + 17).astype(np.int32)
    ids, cnt, _ = oracle.reservation_layout(need + 17, order, page, kv)
    np.testing.assert_array_equal(cnt, (kv + page - 1) // page)   # ceil(n/16) per head
    assert len(set(ids.tolist())) == len(ids) == need              # no page twice
    np.testing.assert_array_equal(ids, order[:need])               # FIFO from the front
    with pytest.raises(RuntimeError):
        oracle.reservation_layout(need - 1, order[:need - 1], page, kv)


def test_reservation_shared_refcounts():
    # shared pages appear once per reader; private pages once
    page, H = 16, 2
    seg = [48, 33]                    # 3 and 2 full pages per head
    chain = np.array([[0, 1], [0, -1], [0, 1], [-1, -1]])
    kv = np.array([[90, 81], [60, 48], [81, 81], [5, 20]], np.int32)
    n = 200
    ids, cnt, segp = oracle.reservation_layout(n, np.arange(n, dtype=np.int32), page, kv, seg, chain)
    sh = set(segp.tolist())
    uses = np.bincount(ids, minlength=n)
    readers = {0: 3, 1: 2}
    for s, full in [(0, 3), (1, 2)]:
        base = sum(H * (seg[k] // page) for k in range(s))
        for p in segp[base:base + H * full]:
            assert uses[p] == readers[s]
    priv = [p for p in ids.tolist() if p not in sh]
    assert len(priv) == len(set(priv))


def test_group_tables_golden():
    for c in gold("group_tables.json")["cases"]:
        t, off, goff = oracle.group_tables(c["group_of_head"], c["G"], c["page_ids"],
                                           np.array(c["head_count"]))
        np.testing.assert_array_equal(t, c["table"])
        np.testing.assert_array_equal(off, c["head_off"])
        np.testing.assert_array_equal(goff, c["group_off"])


def test_radix_example_page_counts():
    g = gold("radix_example.json")
    page = g["page"]
    pin = g["pinned"]
    # Full pages of shared segments (floor), via the layout of one reader per segment.
    for tok, full in pin["shared_full_pages"].items():
        tok = int(tok)
        ids, cnt, segp = oracle.reservation_layout(400, np.arange(400, dtype=np.int32), page,
                                                   np.array([[tok]]), [tok], np.array([[0]]))
        assert len(segp) == full
    # Leaf segments are private pages: ceil.
    for tok, pages in pin["leaf_pages"].items():
        _, cnt, _ = oracle.reservation_layout(400, np.arange(400, dtype=np.int32), page,
                                              np.array([[int(tok)]]))
        assert int(cnt[0, 0]) == pages
    # The page's own sum: 124 + 31 + 5 = 160 (its 124 is the garbled count; see fixture).
    pr = g["printed"]
    assert pr["system_2000"] + pr["docA_500"] + pr["q_80"] == pr["no_tree_total"]


def test_placement_golden_and_bound():
    for c in gold("placement.json")["cases"]:
        np.testing.assert_array_equal(oracle.place_sequences(c["bytes"], c["n_gpus"]), c["gpu"])
    rng = np.random.default_rng(3)
    b = rng.integers(1, 10**6, 300)
    for n in (2, 3, 8):
        g = oracle.place_sequences(b, n)
        load = np.bincount(g, weights=b, minlength=n)
        # LPT: makespan <= mean load + largest single item
        assert load.max() <= b.sum() / n + b.max()


# ---------------------------------------------------------------------------------------
# Decode attention: closed forms, brute force, library routine, invariants.
# ---------------------------------------------------------------------------------------

def _one_head_case(K, V, q, page=16, order=None, scale=None):
    """One sequence, one KV head (G query rows). K, V bf16 bits [n, D]; q bits [G, D]."""
    n, D = K.shape
    G = q.shape[0]
    npg = max(1, -(-n // page))
    order = np.arange(npg + 3)[::-1].copy() if order is None else order
    kp, ids, cnt = scatter_rows([K], page, order, D, num_pages=len(order))
    vp, _, _ = scatter_rows([V], page, order, D, num_pages=len(order))
    table, off = flat_table(ids, cnt)
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    out, lse = oracle.decode(q.reshape(1, G, D), kp, vp, table if len(table) else np.zeros(1, np.int32),
                             off.reshape(1, 1), np.array([[n]], np.int32), scale)
    return out, lse


def test_single_token_returns_v():
    rng = np.random.default_rng(4)
    D = 64
    K, V, q = bf16(rng.normal(size=(1, D))), bf16(rng.normal(size=(1, D))), bf16(rng.normal(size=(3, D)))
    out, lse = _one_head_case(K, V, q)
    np.testing.assert_array_equal(out, np.tile(widen(V), (3, 1)))          # exactly v
    s0 = (widen(q) @ widen(K)[0]) / np.sqrt(D)
    np.testing.assert_allclose(lse, s0, rtol=0, atol=1e-12)                # lse = s_0


def test_identical_keys_give_mean_of_v():
    rng = np.random.default_rng(5)
    D, n = 128, 37
    krow = bf16(rng.normal(size=(1, D)))
    K = np.tile(krow, (n, 1))
    V = bf16(rng.normal(size=(n, D)))
    q = bf16(rng.normal(size=(2, D)))
    out, lse = _one_head_case(K, V, q)
    np.testing.assert_allclose(out, np.tile(widen(V).mean(0), (2, 1)), atol=1e-12)
    s = (widen(q) @ widen(krow)[0]) / np.sqrt(D)
    np.testing.assert_allclose(lse, s + np.log(n), atol=1e-12)


def test_constant_v_returns_v():
    rng = np.random.default_rng(6)
    D, n = 64, 50
    K = bf16(rng.normal(size=(n, D)) * 3)
    vrow = bf16(rng.normal(size=(1, D)))
    out, _ = _one_head_case(K, np.tile(vrow, (n, 1)), bf16(rng.normal(size=(4, D))))
    np.testing.assert_allclose(out, np.tile(widen(vrow), (4, 1)), atol=1e-12)


def test_empty_head():
    D = 64
    K = np.zeros((0, D), np.uint16)
    out, lse = _one_head_case(K, K, bf16(np.ones((2, D))))
    assert (out == 0).all() and np.isneginf(lse).all()


def _sdpa(q, K, V, scale, mask=None):
    """Dense attention by the library routine (torch SDPA, fp64) and its log-sum-exp."""
    qt = torch.from_numpy(q)[None, :, None, :]          # [1, G, 1, D]
    kt = torch.from_numpy(K)[None, None].expand(1, q.shape[0], -1, -1)
    vt = torch.from_numpy(V)[None, None].expand(1, q.shape[0], -1, -1)
    am = None if mask is None else torch.from_numpy(mask)[None, None, None, :]
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, scale=scale)
    s = (torch.from_numpy(q) @ torch.from_numpy(K).T) * scale
    if mask is not None:
        s = s.masked_fill(~torch.from_numpy(mask)[None, :], float("-inf"))
    return out[0, :, 0].numpy(), torch.logsumexp(s, dim=-1).numpy()


def test_full_budget_through_permuted_pages_equals_dense_sdpa():
    rng = np.random.default_rng(7)
    D, n, G = 128, 203, 4
    K, V, q = bf16(rng.normal(size=(n, D))), bf16(rng.normal(size=(n, D))), bf16(rng.normal(size=(G, D)))
    npg = -(-n // 16)
    order = rng.permutation(npg + 5)
    out, lse = _one_head_case(K, V, q, order=order)
    ref, rlse = _sdpa(widen(q), widen(K), widen(V), 1 / np.sqrt(D))
    np.testing.assert_allclose(out, ref, atol=1e-12)
    np.testing.assert_allclose(lse, rlse, atol=1e-12)


def test_brute_force_masked_dense_equals_paged_retained_subset():
    """Full context, seeded retained subset: masked dense attention (−inf on dropped
    positions) equals the paged oracle over only the retained tokens."""
    rng = np.random.default_rng(8)
    D, L, G = 64, 90, 2
    Kf, Vf, q = bf16(rng.normal(size=(L, D))), bf16(rng.normal(size=(L, D))), bf16(rng.normal(size=(G, D)))
    keep = rng.random(L) < 0.4
    keep[rng.integers(L)] = True
    out, lse = _one_head_case(Kf[keep], Vf[keep], q, order=rng.permutation(10))
    ref, rlse = _sdpa(widen(q), widen(Kf), widen(Vf), 1 / np.sqrt(D), mask=keep)
    np.testing.assert_allclose(out, ref, atol=1e-12)
    np.testing.assert_allclose(lse, rlse, atol=1e-12)


def _multi_head_workload(rng, B=3, Hq=8, Hkv=2, D=64, maxn=120, page=16):
    kv = rng.integers(1, maxn, (B, Hkv)).astype(np.int32)
    rows_k = [bf16(rng.normal(size=(int(n), D))) for n in kv.reshape(-1)]
    rows_v = [bf16(rng.normal(size=(int(n), D))) for n in kv.reshape(-1)]
    need = int(((kv + page - 1) // page).sum())
    order = rng.permutation(need + 7)
    kp, ids, cnt = scatter_rows(rows_k, page, order, D, num_pages=need + 7)
    vp, _, _ = scatter_rows(rows_v, page, order, D, num_pages=need + 7)
    table, off = flat_table(ids, cnt)
    q = bf16(rng.normal(size=(B, Hq, D)))
    return dict(q=q, kp=kp, vp=vp, table=table, off=off.reshape(B, Hkv), kv=kv, rows_k=rows_k,
                rows_v=rows_v, D=D, B=B, Hq=Hq, Hkv=Hkv, order=order, page=page)


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (8, 8), (8, 1)])
def test_gqa_mapping_against_per_row_sdpa(Hq, Hkv):
    """Every query row against the library routine on its own KV head's rows: pins the
    contiguous GQA mapping hq -> hq // (Hq/Hkv) and the per-(b, h) table offsets; Hq = Hkv is
    plain multi-head attention (G = 1), Hkv = 1 multi-query."""
    rng = np.random.default_rng(9 + Hkv)
    w = _multi_head_workload(rng, Hq=Hq, Hkv=Hkv)
    out, lse = oracle.decode(w["q"], w["kp"], w["vp"], w["table"], w["off"], w["kv"], 0.125)
    G = w["Hq"] // w["Hkv"]
    for b in range(w["B"]):
        for hq in range(w["Hq"]):
            h = hq // G
            i = b * w["Hkv"] + h
            ref, rl = _sdpa(widen(w["q"][b, hq:hq + 1]), widen(w["rows_k"][i]),
                            widen(w["rows_v"][i]), 0.125)
            np.testing.assert_allclose(out[b * w["Hq"] + hq], ref[0], atol=1e-12)
            np.testing.assert_allclose(lse[b * w["Hq"] + hq], rl[0], atol=1e-12)


def test_permutation_invariance_pages_and_tokens():
    rng = np.random.default_rng(10)
    D, n, G = 64, 77, 2
    K, V, q = bf16(rng.normal(size=(n, D))), bf16(rng.normal(size=(n, D))), bf16(rng.normal(size=(G, D)))
    a, la = _one_head_case(K, V, q, order=rng.permutation(9))
    b, lb = _one_head_case(K, V, q, order=rng.permutation(9))        # different page placement
    perm = rng.permutation(n)
    c, lc = _one_head_case(K[perm], V[perm], q)                        # tokens permuted jointly
    np.testing.assert_allclose(a, b, atol=1e-13)
    np.testing.assert_allclose(a, c, atol=1e-12)
    np.testing.assert_allclose(la, lc, atol=1e-12)
    # transposed operands (K and V swapped) must change the answer
    d, _ = _one_head_case(V, K, q)
    assert np.abs(a - d).max() > 1e-3


def test_split_merge_equals_unsplit():
    """Online-normaliser equivalence: LSE-merging the partial results of any partition of
    each head's tokens reproduces the unsplit result."""
    rng = np.random.default_rng(11)
    w = _multi_head_workload(rng, B=2, Hq=4, Hkv=2, D=64, maxn=200)
    full, flse = oracle.decode(w["q"], w["kp"], w["vp"], w["table"], w["off"], w["kv"], 0.125)
    S = 4
    cuts = np.sort(rng.integers(0, w["kv"][..., None] + 1, (w["B"], w["Hkv"], S - 1)), axis=-1)
    bounds = np.concatenate([np.zeros((w["B"], w["Hkv"], 1), np.int64), cuts,
                             w["kv"][..., None].astype(np.int64)], axis=-1)
    po, pl = [], []
    for j in range(S):
        o, l = oracle.decode(w["q"], w["kp"], w["vp"], w["table"], w["off"], w["kv"], 0.125,
                             tok_lo=bounds[..., j], tok_hi=bounds[..., j + 1])
        po.append(o); pl.append(l)
    out, lse = oracle.lse_merge(np.stack(po), np.stack(pl))
    np.testing.assert_allclose(out, full, atol=1e-12)
    np.testing.assert_allclose(lse, flse, atol=1e-12)


def test_merge_closed_forms():
    rng = np.random.default_rng(12)
    o = rng.normal(size=(2, 3, 8))
    out, lse = oracle.lse_merge(o, np.full((2, 3), 1.7))        # equal weights: the average
    np.testing.assert_allclose(out, o.mean(0), atol=1e-14)
    np.testing.assert_allclose(lse, 1.7 + np.log(2), atol=1e-14)
    pl = np.array([[0.3, -np.inf, -np.inf]]).T.repeat(1, 1).reshape(3, 1)
    out, lse = oracle.lse_merge(o[:, :1].repeat(3, 0)[:3].reshape(3, 1, 8), pl)
    np.testing.assert_allclose(out[0], o[0, 0], atol=1e-14)      # empty splits drop out
    np.testing.assert_allclose(lse, [0.3])
    out, lse = oracle.lse_merge(o[:, :1], np.full((2, 1), -np.inf))
    assert (out == 0).all() and np.isneginf(lse).all()


# ---------------------------------------------------------------------------------------
# Tiered decode and the INT8 quantiser.
# ---------------------------------------------------------------------------------------

def test_quantize_golden():
    for c in gold("quantize_int8.json")["cases"]:
        codes, scale = oracle.quantize_int8(bf16([c["x"]]))
        np.testing.assert_array_equal(codes[0], c["codes"])
        assert float(scale[0]) == c["scale"]


def test_quantize_bounds_and_symmetry():
    x = bf16(np.random.default_rng(13).normal(size=(500, 128)) * 2)
    codes, scale = oracle.quantize_int8(x)
    xf = widen(x)
    assert (np.abs(codes.astype(int)) <= 127).all()
    assert (np.abs(codes).max(1) == 127).all()                          # the max maps to ±127
    err = np.abs(xf - codes * scale[:, None].astype(np.float64))
    assert (err <= scale[:, None] * (0.5 + 1e-5)).all()                 # half a step
    neg = synth.f64_to_bf16_bits(-xf)
    nc, ns = oracle.quantize_int8(neg)
    np.testing.assert_array_equal(nc, -codes)
    np.testing.assert_array_equal(ns, scale)


def test_tiered_equals_untiered_on_exact_values():
    """Values c * 2^-e (|c| <= 127, per-token e, different for K and V) are exact both in
    bf16 and as INT8 code * scale, so the tiered oracle (slow INT8 + fast bf16) must equal the
    untiered oracle on the same rows."""
    rng = np.random.default_rng(14)
    B, Hq, Hkv, D, page = 2, 4, 2, 64, 16
    kv = np.array([[70, 33], [16, 100]], np.int32)
    fast = np.array([[20, 33], [0, 17]], np.int32)
    q = bf16(rng.normal(size=(B, Hq, D)))
    ck = [rng.integers(-127, 128, (int(n), D)) for n in kv.reshape(-1)]
    cv = [rng.integers(-127, 128, (int(n), D)) for n in kv.reshape(-1)]
    # per-token power-of-two scales, different for K and V
    sk = [2.0 ** -rng.integers(3, 7, int(n)) for n in kv.reshape(-1)]
    sv = [2.0 ** -rng.integers(2, 9, int(n)) for n in kv.reshape(-1)]
    rows_k = [bf16(c * s[:, None]) for c, s in zip(ck, sk)]
    rows_v = [bf16(c * s[:, None]) for c, s in zip(cv, sv)]
    need = int(((kv + page - 1) // page).sum())
    order = rng.permutation(need + 3)
    kp, ids, cnt = scatter_rows(rows_k, page, order, D, num_pages=need + 3)
    vp, _, _ = scatter_rows(rows_v, page, order, D, num_pages=need + 3)
    t, off = flat_table(ids, cnt)
    ref, rlse = oracle.decode(q, kp, vp, t, off.reshape(B, Hkv), kv, 0.125)

    slow_k, slow_v, fast_k, fast_v, slow_sk, slow_sv = [], [], [], [], [], []
    for i, n in enumerate(kv.reshape(-1)):
        f = min(int(fast.reshape(-1)[i]), int(n))
        slow_k.append(ck[i][:n - f]); slow_v.append(cv[i][:n - f])
        slow_sk.append(sk[i][:n - f]); slow_sv.append(sv[i][:n - f])
        fast_k.append(rows_k[i][n - f:]); fast_v.append(rows_v[i][n - f:])

    def scatter_i8(rows, scales, order):
        counts = [-(-r.shape[0] // page) for r in rows]
        P = sum(counts) + 2
        pool = np.zeros((P, page, D), np.int8)
        scl = np.zeros((P, page), np.float32)
        ids, k = [], 0
        for r, sc, c in zip(rows, scales, counts):
            for p in range(c):
                pid = int(order[k]); k += 1; ids.append(pid)
                ch = r[p * page:(p + 1) * page]
                pool[pid, :len(ch)] = ch
                scl[pid, :len(ch)] = sc[p * page:(p + 1) * page]
        return pool, scl, np.asarray(ids, np.int32), np.asarray(counts, np.int32)

    ns = sum(-(-r.shape[0] // page) for r in slow_k)
    so = rng.permutation(ns + 2)
    kq, ks, sids, scnt = scatter_i8(slow_k, slow_sk, so)
    vq, vs, _, _ = scatter_i8(slow_v, slow_sv, so)
    nf = sum(-(-r.shape[0] // page) for r in fast_k)
    fo = rng.permutation(nf + 2)
    kf, fids, fcnt = scatter_rows(fast_k, page, fo, D, num_pages=nf + 2)
    vf, _, _ = scatter_rows(fast_v, page, fo, D, num_pages=nf + 2)
    st, soff = flat_table(sids, scnt)
    ft, foff = flat_table(fids, fcnt)
    out, lse = oracle.tiered_decode(q, kq, vq, ks, vs, st if len(st) else np.zeros(1, np.int32),
                                    soff.reshape(B, Hkv), kf, vf, ft, foff.reshape(B, Hkv), kv,
                                    fast, 0.125)
    np.testing.assert_allclose(out, ref, atol=1e-12)
    np.testing.assert_allclose(lse, rlse, atol=1e-12)


# ---------------------------------------------------------------------------------------
# The INT4 slow-tier quantiser: hand-worked rows and packed bytes, bounds, symmetry, and the
# exact dequantisation of values c * 2^-e (|c| <= 7) through the tiered decode.
# ---------------------------------------------------------------------------------------

def test_quantize_int4_golden():
    for c in gold("quantize_int4.json")["cases"]:
        packed, scale = oracle.quantize_int4(bf16([c["x"]]))
        np.testing.assert_array_equal(packed[0], c["packed"])
        np.testing.assert_array_equal(oracle.unpack_int4(packed)[0], c["codes"])
        assert float(scale[0]) == c["scale"]


def test_quantize_int4_bounds_and_symmetry():
    x = bf16(np.random.default_rng(23).normal(size=(500, 128)) * 2)
    packed, scale = oracle.quantize_int4(x)
    assert packed.shape == (500, 64)
    codes = oracle.unpack_int4(packed).astype(int)
    xf = widen(x)
    assert (np.abs(codes) <= 7).all()
    assert (np.abs(codes).max(1) == 7).all()                            # the max maps to ±7
    err = np.abs(xf - codes * scale[:, None].astype(np.float64))
    assert (err <= scale[:, None] * (0.5 + 1e-5)).all()                 # half a step
    assert ((packed & 0xF) != 0).all() and ((packed >> 4) != 0).all()   # nibble 0 (= -8) unused
    nc = oracle.unpack_int4(oracle.quantize_int4(synth.f64_to_bf16_bits(-xf))[0])
    np.testing.assert_array_equal(nc, -codes)


def test_int4_tier_equals_untiered_on_exact_values():
    """Rows c * 2^-e with |c| <= 7 and a 7 in every row quantise exactly (scale 2^-e): the
    INT4 quantiser returns c, and the tiered decode of the unpacked INT4 tier equals the
    untiered decode of the bf16 rows."""
    rng = np.random.default_rng(24)
    B, Hq, Hkv, D, page = 1, 4, 2, 64, 16
    kv = np.array([[50, 37]], np.int32)
    fast = np.array([[18, 5]], np.int32)
    q = bf16(rng.normal(size=(B, Hq, D)))
    rows_k, rows_v = [], []
    for n in kv.reshape(-1):
        for rows in (rows_k, rows_v):
            c = rng.integers(-7, 8, (int(n), D))
            c[np.arange(int(n)), rng.integers(0, D, int(n))] = rng.choice([-7, 7], int(n))
            e = rng.integers(2, 9, int(n))
            rows.append(bf16(c * 2.0 ** -e[:, None]))
    need = int(((kv + page - 1) // page).sum())
    order = rng.permutation(need)
    kp, ids, cnt = scatter_rows(rows_k, page, order, D, num_pages=need)
    vp, _, _ = scatter_rows(rows_v, page, order, D, num_pages=need)
    t, off = flat_table(ids, cnt)
    ref, rlse = oracle.decode(q, kp, vp, t, off.reshape(B, Hkv), kv, 0.125)
    # slow tier = the first n - f tokens of each head, quantised to INT4 page by page
    slow_k = [r[:n - f] for r, n, f in zip(rows_k, kv.reshape(-1), fast.reshape(-1))]
    slow_v = [r[:n - f] for r, n, f in zip(rows_v, kv.reshape(-1), fast.reshape(-1))]
    fast_k = [r[n - f:] for r, n, f in zip(rows_k, kv.reshape(-1), fast.reshape(-1))]
    fast_v = [r[n - f:] for r, n, f in zip(rows_v, kv.reshape(-1), fast.reshape(-1))]
    ns = sum(-(-r.shape[0] // page) for r in slow_k)
    so = rng.permutation(ns)
    kb, sids, scnt = scatter_rows(slow_k, page, so, D, num_pages=ns)
    vb, _, _ = scatter_rows(slow_v, page, so, D, num_pages=ns)
    kpk, ks = oracle.quantize_int4(kb)
    vpk, vs = oracle.quantize_int4(vb)
    kq, vq = oracle.unpack_int4(kpk), oracle.unpack_int4(vpk)
    np.testing.assert_array_equal(kq * ks[..., None].astype(np.float64), widen(kb))   # exact
    nf = sum(-(-r.shape[0] // page) for r in fast_k)
    fo = rng.permutation(nf)
    kf, fids, fcnt = scatter_rows(fast_k, page, fo, D, num_pages=nf)
    vf, _, _ = scatter_rows(fast_v, page, fo, D, num_pages=nf)
    st, soff = flat_table(sids, scnt)
    ft, foff = flat_table(fids, fcnt)
    out, lse = oracle.tiered_decode(q, kq, vq, ks, vs, st, soff.reshape(B, Hkv), kf, vf, ft,
                                    foff.reshape(B, Hkv), kv, fast, 0.125)
    np.testing.assert_allclose(out, ref, atol=1e-12)
    np.testing.assert_allclose(lse, rlse, atol=1e-12)


# ---------------------------------------------------------------------------------------
# Decode-step write path (sink + recent, H2O): hand-worked cases, closed forms, invariants.
# ---------------------------------------------------------------------------------------

def _run_sink_recent(budget, sink, kv_len, slot_pos, new_positions):
    pos = list(slot_pos) + [-1] * (budget - len(slot_pos))
    n = kv_len
    slots = []
    for p in new_positions:
        s = oracle.sink_recent_slot(budget, sink, n, np.array(pos[:max(n, 1)], np.int32))
        assert 0 <= s < budget, (budget, sink, n)    # a head with budget >= 1 always takes a slot
        slots.append(s)
        pos[s] = p
        n = max(n, s + 1)
    return slots, pos[:n]


def test_sink_recent_golden():
    for c in gold("write_path.json")["sink_recent"]:
        slots, final = _run_sink_recent(c["budget"], c["sink"], c["kv_len"], c["slot_pos"], c["new_pos"])
        assert slots == c["slots"], c["work"]
        assert final == c["final_pos"], c["work"]


def test_sink_recent_sinks_never_fill_the_budget():
    """At most budget - 1 sinks: with sink >= budget one slot still turns over (hand-worked:
    budget 3, sink 5, positions 0, 1, 2 in slots 0-2; sinks are positions 0 and 1, so the new
    position 3 replaces position 2 in slot 2, then position 4 replaces 3 in slot 2)."""
    slots, final = _run_sink_recent(3, 5, 3, [0, 1, 2], [3, 4])
    assert slots == [2, 2] and final == [0, 1, 4]
    assert oracle.sink_recent_slot(1, 3, 1, np.array([7], np.int32)) == 0   # budget 1: no sink


def test_sink_recent_keeps_first_and_last_tokens():
    """Closed form of the rule the pages describe: after any number of steps a full head holds
    exactly the first s positions and the last budget - s positions."""
    rng = np.random.default_rng(40)
    for _ in range(200):
        budget = int(rng.integers(1, 40))
        sink = int(rng.integers(0, 6))
        L = int(rng.integers(budget, 200))
        s = min(sink, budget - 1)
        start = list(range(s)) + list(range(L - (budget - s), L))
        T = int(rng.integers(0, 120))
        _, final = _run_sink_recent(budget, sink, budget, start, range(L, L + T))
        want = set(range(s)) | set(range(L + T - (budget - s), L + T))
        assert sorted(final) == sorted(want)


def test_h2o_golden():
    for c in gold("write_path.json")["h2o"]:
        got = oracle.h2o_victim(c["budget"], c["recent"], c["kv_len"], np.array(c["slot_pos"], np.int32),
                                np.array(c["score"], np.float32), c["new_pos"])
        assert got == c["slot"], c["work"]


def test_h2o_with_age_scores_is_a_sliding_window():
    """Special case: when every token's score equals its position, the lowest-scored candidate
    is the oldest token, so H2O reduces to a sliding window of the last `budget` positions."""
    rng = np.random.default_rng(41)
    for _ in range(100):
        budget = int(rng.integers(1, 30))
        recent = int(rng.integers(0, 40))
        L = int(rng.integers(budget, 100))
        pos = np.arange(L - budget, L, dtype=np.int32)
        rng.shuffle(pos)
        for p in range(L, L + int(rng.integers(1, 80))):
            v = oracle.h2o_victim(budget, recent, budget, pos, pos.astype(np.float32), p)
            pos[v] = p
        assert sorted(pos.tolist()) == list(range(p + 1 - budget, p + 1))


def test_h2o_never_evicts_the_recent_window():
    rng = np.random.default_rng(42)
    for _ in range(300):
        budget = int(rng.integers(2, 50))
        recent = int(rng.integers(0, budget))
        L = budget + int(rng.integers(0, 100))
        pos = np.sort(rng.choice(L, size=budget, replace=False)).astype(np.int32)
        pos[-min(recent, budget):] = np.arange(L - min(recent, budget), L) if recent else pos[-1:]
        pos = np.unique(pos)
        if pos.size < budget:
            continue
        score = rng.random(budget).astype(np.float32)
        v = oracle.h2o_victim(budget, recent, budget, pos, score, L)
        older = pos < L - recent
        if older.any():
            assert older[v]
            assert score[v] == score[older].min()
            assert v == np.flatnonzero(older & (score == score[older].min()))[0]
        else:
            assert pos[v] == pos.min()


def test_token_scores_logsumexp_equals_decode_lse():
    """The per-token scores tie to the (pinned) decode: ln sum_t exp(s_t) is its lse."""
    sp = synth.small(2)
    from tests import _oracle_side as ors
    lay = ors.layout(sp, 0)
    q = synth.q_bits(sp)
    k = synth.pool_bits(sp, "k", lay.num_pages)
    s = oracle.token_scores(q, k, lay.table, lay.head_off, lay.kv_len, sp.scale, lay.table.size)
    _, ref_lse = ors.reference(sp, lay, 0)
    G = sp.Hq // sp.Hkv
    for b in range(sp.B):
        for h in range(sp.Hkv):
            n = int(lay.kv_len[b, h])
            base = int(lay.head_off[b, h]) * sp.page
            st = s[base:base + n]
            assert not np.isnan(st).any()
            for g in range(G):
                want = ref_lse[b * sp.Hq + h * G + g]
                got = np.logaddexp.reduce(st[:, g]) if n else -np.inf
                assert got == pytest.approx(want, abs=1e-9)


def test_h2o_accumulate_adds_one_per_query_head():
    """Each query head's attention sums to 1 over the retained tokens, so the scores of a head
    grow by G in total per step."""
    rng = np.random.default_rng(43)
    for n, G in ((1, 1), (7, 4), (300, 8)):
        s = rng.normal(size=(n, G)) * 3
        lse = np.logaddexp.reduce(s, axis=0)
        sc0 = (rng.random(n) * 4).astype(np.float32)
        sc1 = oracle.h2o_accumulate(s, lse, sc0)
        assert (sc1 >= sc0).all()
        inc = sc1.astype(np.float64) - sc0.astype(np.float64)
        assert inc.sum() == pytest.approx(G, abs=n * 4 * 2.0 ** -23)


# ---------------------------------------------------------------------------------------
# Tier migration (fast window -> INT8 tier): hand-worked steps and the tier invariants.
# ---------------------------------------------------------------------------------------

def test_tier_step_hand_worked():
    """cap 3: positions 0, 1, 2 fill fast slots 0, 1, 2; position 3 moves position 0 to slow
    index 0 and takes slot 0; position 4 moves 1 (slot 1); position 5 moves 2 (slot 2); 6 moves
    3 (slot 0)."""
    n, f = 0, 0
    got = []
    for _ in range(7):
        got.append(oracle.tier_step(n, f, 3, 100))
        n, f = n + 1, min(f + 1, 3)
    assert got == [(0, -1), (1, -1), (2, -1), (0, 0), (1, 1), (2, 2), (0, 3)]
    assert oracle.tier_step(10, 2, 3, 100) == (-1, -1)     # not full, yet older tokens exist
    assert oracle.tier_step(10, 3, 3, 7) == (-1, -1)       # no reserved slow slot for position 7
    assert oracle.tier_step(10, 3, 3, 8) == (1, 7)


def test_tier_step_keeps_recent_fast_and_older_slow():
    rng = np.random.default_rng(45)
    for _ in range(60):
        cap = int(rng.integers(1, 40))
        fast = {}
        slow = []
        n, f = 0, 0
        for _ in range(int(rng.integers(1, 200))):
            fs, si = oracle.tier_step(n, f, cap, 10**6)
            assert fs >= 0
            if si >= 0:
                assert fast[fs] == si                   # the oldest fast token leaves
                slow.append(si)
            fast[fs] = n
            n, f = n + 1, min(f + 1, cap)
        assert sorted(fast.values()) == list(range(n - f, n))
        assert all(s_ == p % cap for s_, p in fast.items())
        assert slow == list(range(n - f))


# ---------------------------------------------------------------------------------------
# SplitZip codec: hand-worked streams, lossless round trip, codebook and escapes by brute force.
# ---------------------------------------------------------------------------------------

def _bf16_specials(rng, n):
    x = rng.integers(0, 1 << 16, n).astype(np.uint16)               # any bit pattern
    special = np.array([0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC0, 0xFFC1, 0x0001, 0x807F,
                        0x3F80, 0x7F7F], np.uint16)
    x[rng.integers(0, n, min(n, 40))] = rng.choice(special, min(n, 40))
    return x


def test_splitzip_golden():
    for c in gold("splitzip.json")["cases"]:
        x = np.array(c["x"], np.uint16)
        cb, sm, codes, pos, exp = oracle.splitzip_encode(x)
        assert cb[:len(c["codebook_head"])].tolist() == c["codebook_head"], c["work"]
        assert sm.tolist() == c["sm"] and codes.tolist() == c["codes"], c["work"]
        assert pos.tolist() == c["esc_pos"] and exp.tolist() == c["esc_exp"], c["work"]
        np.testing.assert_array_equal(oracle.splitzip_decode(x.size, cb, sm, codes, pos, exp), x)


@pytest.mark.parametrize("n", [0, 1, 2, 7, 1000, 65537])
def test_splitzip_round_trip_is_lossless(n):
    rng = np.random.default_rng(47 + n)
    for x in (_bf16_specials(rng, n), bf16(rng.normal(size=n) * 3) if n else np.zeros(0, np.uint16)):
        cb, sm, codes, pos, exp = oracle.splitzip_encode(x)
        np.testing.assert_array_equal(oracle.splitzip_decode(x.size, cb, sm, codes, pos, exp), x)


def test_splitzip_codebook_and_escapes_by_brute_force():
    rng = np.random.default_rng(48)
    for x in (bf16(rng.normal(size=5000)), _bf16_specials(rng, 3000), bf16(rng.standard_cauchy(4000))):
        cb, sm, codes, pos, exp = oracle.splitzip_encode(x)
        e = (x >> 7) & 0xFF
        counts = np.bincount(e, minlength=256)
        order = np.lexsort((np.arange(256), -counts))               # count desc, exponent asc
        np.testing.assert_array_equal(cb, order[:16])
        esc = np.flatnonzero(~np.isin(e, cb))
        np.testing.assert_array_equal(pos, esc)
        np.testing.assert_array_equal(exp, e[esc])
        assert (sm == (((x >> 15) << 7) | (x & 0x7F))).all()
        # normal data: the top 16 exponents cover almost everything (the page's premise)
    xn = bf16(rng.normal(size=100000))
    assert oracle.splitzip_encode(xn)[3].size < 0.01 * xn.size
