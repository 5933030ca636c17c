"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test checks the oracle against something it does not compute itself:
a hand-worked example of the merge formula (golden file), high-precision
brute force with Python's decimal module, closed forms, special cases that
reduce to scipy's softmax/logsumexp, exact algebraic identities of the merge
(partition invariance, empty-partner identity), and the decision rules of the
reuse policy enumerated by hand.  ``test_planted_mistakes_are_caught`` checks
that plausible slips in the oracle make these pins fail.

Source: "FlashBlock: Attention Caching for Efficient Long-Context Block
Diffusion", gist.science summary, sections "Mécanisme Central" and
"Stratégies de Réutilisation Adaptatives".
"""
import decimal
import json
import math
import os

import numpy as np
import pytest
import scipy.special

from oracle import flashblock_oracle as orc
from block_diffusion_attention_flashblock_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "merge_worked_example.json")


def _num(x):
    """Parse the golden file's exact forms: numbers, 'ln k', 'c + ln k', '-inf'."""
    if isinstance(x, (int, float)):
        return float(x)
    x = x.strip()
    if x == "-inf":
        return -math.inf
    total = 0.0
    for term in x.split("+"):
        term = term.strip()
        if term.startswith("ln "):
            total += math.log(float(term[3:]))
        else:
            total += float(term)
    return total


def _arr(a):
    return np.array([[_num(v) for v in row] for row in a]) if isinstance(a[0], list) \
        else np.array([_num(v) for v in a])


# ---------------------------------------------------------------- golden ---
def check_golden(mod=orc):
    g = json.load(open(GOLDEN))
    for c in g["merge_cases"]:
        A, L = mod.merge([(np.array([_arr(c["A_out"])]), np.array([_num(c["L_out"])])),
                          (np.array([_arr(c["A_in"])]), np.array([_num(c["L_in"])]))])
        np.testing.assert_allclose(A[0], _arr(c["A"]), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(L[0], _num(c["L"]), rtol=1e-14)
    for c in g["attention_cases"]:
        A, L = mod.attention_part(_arr(c["q"]), _arr(c["k"]), _arr(c["v"]), c["scale"])
        np.testing.assert_allclose(A, _arr(c["A"]), rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(L, _arr(c["L"]), rtol=1e-13)


def test_golden_worked_examples():
    check_golden()


# ---------------------------------------------------------- brute force ---
def _decimal_attention(q, k, v, scale):
    """Direct sum with 40 significant digits and no max shift (tiny inputs)."""
    decimal.getcontext().prec = 40
    D = decimal.Decimal
    out_A, out_L = [], []
    for qi in q:
        e = []
        for kj in k:
            s = D(repr(float(scale))) * sum(D(repr(float(a))) * D(repr(float(b)))
                                            for a, b in zip(qi, kj))
            e.append(s.exp())
        Z = sum(e)
        out_A.append([float(sum(ej * D(repr(float(vj[d]))) for ej, vj in zip(e, v)) / Z)
                      for d in range(v.shape[1])])
        out_L.append(float(Z.ln()))
    return np.array(out_A), np.array(out_L)


def check_brute_force(mod=orc, seed=0):
    rng = np.random.default_rng(seed)
    for m in (1, 2, 5, 8):
        q = rng.uniform(-1, 1, (3, 4)); k = rng.uniform(-1.5, 1.5, (m, 4))
        v = rng.standard_normal((m, 4))
        A, L = mod.attention_part(q, k, v, 0.7)
        A_ref, L_ref = _decimal_attention(q, k, v, 0.7)
        np.testing.assert_allclose(A, A_ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(L, L_ref, rtol=1e-13, atol=1e-13)


def test_brute_force_decimal():
    check_brute_force()


# -------------------------------------------------------- library special ---
def check_softmax_special_case(mod=orc):
    """K = V = I_D: scores are scale*q itself, A is softmax(scale q), L = logsumexp."""
    rng = np.random.default_rng(1)
    D = 16
    q = rng.standard_normal((5, D)) * 3.0
    eye = np.eye(D)
    A, L = mod.attention_part(q, eye, eye, 0.25)
    np.testing.assert_allclose(A, scipy.special.softmax(0.25 * q, axis=1), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(L, scipy.special.logsumexp(0.25 * q, axis=1), rtol=1e-13)
    # non-square: V = ones column block -> each softmax row sums to one
    A1, _ = mod.attention_part(q, eye, np.ones((D, 3)), 0.25)
    np.testing.assert_allclose(A1, np.ones((5, 3)), rtol=1e-13)


def test_softmax_special_case():
    check_softmax_special_case()


# ---------------------------------------------------------- closed forms ---
def check_closed_forms(mod=orc):
    rng = np.random.default_rng(2)
    D = 8
    # one key: A = v, L = s (s = scale * a * b with q = a e0, k = b e0)
    q = np.zeros((1, D)); q[0, 0] = 1.5
    k = np.zeros((1, D)); k[0, 0] = -2.0
    v = rng.standard_normal((1, D))
    A, L = mod.attention_part(q, k, v, 0.5)
    np.testing.assert_allclose(A, v, rtol=1e-15)
    np.testing.assert_allclose(L, [0.5 * 1.5 * -2.0], rtol=1e-15)
    # q = 0: uniform weights, A = mean(V), L = log m
    m = 37
    A, L = mod.attention_part(np.zeros((2, D)), rng.standard_normal((m, D)),
                              (V := rng.standard_normal((m, D))), 0.3)
    np.testing.assert_allclose(A, np.tile(V.mean(0), (2, 1)), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(L, [math.log(m)] * 2, rtol=1e-14)
    # identical keys: A = mean(V), L = s + log m
    kk = np.zeros((m, D)); kk[:, 1] = 2.0
    qq = np.zeros((1, D)); qq[0, 1] = 0.75
    A, L = mod.attention_part(qq, kk, V, 1.0)
    np.testing.assert_allclose(A[0], V.mean(0), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(L, [1.5 + math.log(m)], rtol=1e-14)
    # empty key set
    A, L = mod.attention_part(np.ones((3, D)), np.zeros((0, D)), np.zeros((0, D)), 1.0)
    assert np.all(A == 0) and np.all(np.isneginf(L))


def test_closed_forms():
    check_closed_forms()


# ------------------------------------------------------- merge identities ---
def check_partition_invariance(mod=orc, seed=3):
    rng = np.random.default_rng(seed)
    n, m, D = 6, 60, 16
    q = rng.standard_normal((n, D)) * 2
    k = rng.standard_normal((m, D)); v = rng.standard_normal((m, D))
    A_full, L_full = mod.attention_part(q, k, v, 0.4)
    for trial in range(20):
        nparts = rng.integers(1, 6)
        label = rng.integers(0, nparts, m)
        parts = [mod.attention_part(q, k[label == p], v[label == p], 0.4) for p in range(nparts)]
        order = rng.permutation(nparts)
        A, L = mod.merge([parts[i] for i in order])
        np.testing.assert_allclose(A, A_full, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(L, L_full, rtol=1e-13, atol=1e-13)
        if nparts >= 3:   # grouping: merge(merge(p0, p1), rest...) == flat merge
            A2, L2 = mod.merge([mod.merge(parts[:2])] + parts[2:])
            np.testing.assert_allclose(A2, A_full, rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(L2, L_full, rtol=1e-13, atol=1e-13)


def test_partition_invariance():
    check_partition_invariance()


def test_empty_partner_is_bit_exact_identity():
    rng = np.random.default_rng(4)
    A = rng.standard_normal((5, 8)); L = rng.standard_normal(5) * 10
    empty = (np.zeros((5, 8)), np.full(5, -np.inf))
    for parts in ([(A, L), empty], [empty, (A, L)], [empty, (A, L), empty]):
        A2, L2 = orc.merge(parts)
        assert np.array_equal(A2, A) and np.array_equal(L2, L)
    A3, L3 = orc.merge([empty, empty])
    assert np.all(A3 == 0) and np.all(np.isneginf(L3))


def test_merge_symmetric():
    rng = np.random.default_rng(5)
    p1 = (rng.standard_normal((4, 8)), rng.standard_normal(4))
    p2 = (rng.standard_normal((4, 8)), rng.standard_normal(4))
    A12, L12 = orc.merge([p1, p2]); A21, L21 = orc.merge([p2, p1])
    np.testing.assert_allclose(A12, A21, rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(L12, L21, rtol=1e-15)


# -------------------------------------------------------------------- GQA ---
def test_gqa_grouping_and_expansion():
    rng = np.random.default_rng(6)
    B, Hq, Hkv, Nb, D, Lp = 2, 8, 2, 5, 8, 30
    Q = rng.standard_normal((B, Hq, Nb, D))
    Kp = rng.standard_normal((B, Hkv, Lp, D))
    # V of KV head g is the constant g: every query head of group g reads g
    Vp = np.zeros((B, Hkv, Lp, D)); Vp[:, 1] = 1.0
    A, _ = orc.outblock(Q, Kp, Vp, Lp, 0.3)
    assert np.allclose(A[:, :4], 0.0) and np.allclose(A[:, 4:], 1.0)
    # expanding KV heads to Hq (MHA) gives the same result
    Vp = rng.standard_normal((B, Hkv, Lp, D))
    A1, L1 = orc.outblock(Q, Kp, Vp, Lp, 0.3)
    A2, L2 = orc.outblock(Q, np.repeat(Kp, 4, axis=1), np.repeat(Vp, 4, axis=1), Lp, 0.3)
    np.testing.assert_array_equal(A1, A2); np.testing.assert_array_equal(L1, L2)


# ----------------------------------------------------------------- policy ---
def _tiny(**kw):
    spec = wl.get_spec("tiny_f32", **kw)
    return spec, wl.Workload(spec)


def _run(spec, work, tau, gamma=None, sel_fn=None):
    kp, vp = work.prefix_kv()
    kp64, vp64 = orc.to64(kp), orc.to64(vp)
    o = orc.FlashBlockOracle(spec.B, spec.Hq, spec.Hkv, spec.D, spec.Nb, gamma=gamma)
    res = []
    for st in work.schedule():
        if st.step == 0:
            o.begin_block()
        r = o.step(orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin), kp64, vp64,
                   st.prefix_len, st.M, tau, None if st.sel is None else st.sel.numpy())
        res.append((st, r))
        if st.last_in_block:
            kp64, vp64, _ = orc.kv_append(kp64, vp64, st.prefix_len, orc.to64(st.kin), orc.to64(st.vin))
    return res, kp64, vp64


def _full(st, kp64, vp64, scale):
    return orc.full_attention(orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin),
                              kp64, vp64, st.prefix_len, scale)


def test_tau_zero_is_full_attention():
    spec, work = _tiny(blocks=2, steps=3)
    kp, vp = work.prefix_kv(); kp64, vp64 = orc.to64(kp), orc.to64(vp)
    res, _, _ = _run(spec, work, tau=0)
    for st, r in res:
        assert r.recompute
        A, L = orc.full_attention(orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin),
                                  kp64, vp64, st.prefix_len, 1 / 8)
        np.testing.assert_allclose(r.o, A, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(r.lse, L, rtol=1e-12)
        if st.last_in_block:
            kp64, vp64, _ = orc.kv_append(kp64, vp64, st.prefix_len, orc.to64(st.kin), orc.to64(st.vin))


def test_tau_infinite_reuses_step0_cache():
    spec, work = _tiny(steps=4)
    kp, vp = work.prefix_kv(); kp64, vp64 = orc.to64(kp), orc.to64(vp)
    res, _, _ = _run(spec, work, tau=None)
    q0 = orc.to64(res[0][0].q)
    A0, L0 = orc.outblock(q0, kp64, vp64, spec.prefix0, 1 / 8)
    for st, r in res:
        assert r.recompute == (st.step == 0)
        Ai, Li = orc.inblock(orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin), 1 / 8)
        A, L = orc.merge([(A0, L0), (Ai, Li)])
        np.testing.assert_allclose(r.o, A, rtol=1e-12, atol=1e-13)


def test_tau_decisions_enumerated():
    spec, work = _tiny(steps=4)
    res, _, _ = _run(spec, work, tau=spec.tau)
    Ms = [st.M for st, _ in res]
    expect = [True] + [M >= spec.tau for M in Ms[1:]]     # strict M < tau reuses
    assert [r.recompute for _, r in res] == expect
    # the same rule after the tie M == tau: recompute
    o = orc.FlashBlockOracle(1, 1, 1, 4, 2)
    z = np.zeros((1, 1, 2, 4)); kp = np.ones((1, 1, 3, 4))
    o.begin_block()
    assert o.step(z, z, z, kp, kp, 3, 0, 2).recompute
    assert not o.step(z, z, z, kp, kp, 3, 1, 2).recompute
    assert o.step(z, z, z, kp, kp, 3, 2, 2).recompute
    o.begin_block()
    assert o.step(z, z, z, kp, kp, 3, 0, 2).recompute     # new block forces a full step


def test_changed_key_set_recomputes():
    """A cached part is attention over one block-external key set: after the
    prefix grows (without a new block) or the selection changes, the step
    recomputes even with tau off, and equals exact full attention over the
    new prefix plus the block (tau off would otherwise reuse the stale part)."""
    spec, work = _tiny(steps=2)
    kp, vp = work.prefix_kv(); kp64, vp64 = orc.to64(kp), orc.to64(vp)
    steps = list(work.schedule())
    o = orc.FlashBlockOracle(spec.B, spec.Hq, spec.Hkv, spec.D, spec.Nb)
    st = steps[0]
    q, kin, vin = orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin)
    assert o.step(q, kin, vin, kp64, vp64, 200, 0, None).recompute
    assert not o.step(q, kin, vin, kp64, vp64, 200, 0, None).recompute   # same set: reuse
    r = o.step(q, kin, vin, kp64, vp64, 256, 0, None)                    # the prefix grew
    assert r.recompute
    A, L = orc.full_attention(q, kin, vin, kp64, vp64, 256, 1 / 8)
    np.testing.assert_allclose(r.o, A, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(r.lse, L, rtol=1e-12)
    # sparse: a different selection over the same prefix is a different residual set
    sel_a = np.tile(np.arange(0, 256, 4, dtype=np.int32), (1, spec.Hq, 1))
    sel_b = np.tile(np.arange(1, 256, 4, dtype=np.int32), (1, spec.Hq, 1))
    o.begin_block()
    assert o.step(q, kin, vin, kp64, vp64, 256, 0, None, sel_a).recompute
    assert not o.step(q, kin, vin, kp64, vp64, 256, 0, None, sel_a.copy()).recompute
    r = o.step(q, kin, vin, kp64, vp64, 256, 0, None, sel_b)
    assert r.recompute
    A, L = orc.full_attention(q, kin, vin, kp64, vp64, 256, 1 / 8)
    np.testing.assert_allclose(r.o, A, rtol=1e-11, atol=1e-12)


# ------------------------------------------------- active-query subsets ---
def _run_active(spec, work, tau, all_active=False):
    kp, vp = work.prefix_kv()
    kp64, vp64 = orc.to64(kp), orc.to64(vp)
    o = orc.FlashBlockOracle(spec.B, spec.Hq, spec.Hkv, spec.D, spec.Nb)
    res = []
    for st in work.schedule():
        if st.step == 0:
            o.begin_block()
        act = np.tile(np.arange(spec.Nb), (spec.B, 1)) if all_active else st.active.numpy()
        r = o.step(orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin), kp64, vp64, st.prefix_len, st.M, tau,
                   active=act)
        res.append((st, r, (kp64, vp64)))
        if st.last_in_block:
            kp64, vp64, _ = orc.kv_append(kp64, vp64, st.prefix_len, orc.to64(st.kin), orc.to64(st.vin))
    return res


def _tiny_lock(**kw):
    return _tiny(lock_rate=0.3, steps=5, **kw)


def test_active_all_positions_is_the_dense_step():
    """Every position active: the subset step is the dense step."""
    spec, work = _tiny_lock(blocks=2)
    dense, _, _ = _run(spec, work, tau=spec.tau)
    sub = _run_active(spec, work, tau=spec.tau, all_active=True)
    for (st, rd), (_, ra, _) in zip(dense, sub):
        assert rd.recompute == ra.recompute
        np.testing.assert_allclose(ra.o, rd.o, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(ra.lse, rd.lse, rtol=1e-13)


def test_active_rows_of_full_steps_are_full_attention_and_locked_rows_keep_their_output():
    """tau = 0 (every step full): each active row is exact attention over the
    prefix and all block keys (locked tokens' keys included); each locked
    position keeps, bit for bit, its output of the previous step."""
    spec, work = _tiny_lock()
    res = _run_active(spec, work, tau=0)
    prev = None
    for st, r, (kp64, vp64) in res:
        assert r.recompute
        A, L = orc.full_attention(orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin), kp64, vp64,
                                  st.prefix_len, 1 / 8)
        rows = st.active.numpy()[0]
        assert 0 < len(rows) <= spec.Nb
        np.testing.assert_allclose(r.o[:, :, rows], A[:, :, rows], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(r.lse[:, :, rows], L[:, :, rows], rtol=1e-12)
        locked = np.setdiff1d(np.arange(spec.Nb), rows)
        if prev is None:
            assert len(locked) == 0
        else:
            assert np.array_equal(r.o[:, :, locked], prev.o[:, :, locked])
            assert np.array_equal(r.lse[:, :, locked], prev.lse[:, :, locked])
        prev = r


def test_active_reuse_rows_merge_the_block_start_cache():
    """tau off: only step 0 computes the block-external part; an active row at
    step s merges its step-0 cached part with fresh in-block attention."""
    spec, work = _tiny_lock()
    res = _run_active(spec, work, tau=None)
    st0, _, (kp64, vp64) = res[0]
    A0, L0 = orc.outblock(orc.to64(st0.q), kp64, vp64, st0.prefix_len, 1 / 8)
    for st, r, _ in res:
        assert r.recompute == (st.step == 0)
        rows = st.active.numpy()[0]
        Ai, Li = orc.inblock(orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin), 1 / 8)
        A, L = orc.merge([(A0, L0), (Ai, Li)])
        np.testing.assert_allclose(r.o[:, :, rows], A[:, :, rows], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(r.lse[:, :, rows], L[:, :, rows], rtol=1e-12)


def test_active_sets_only_shrink():
    spec, work = _tiny_lock()
    steps = list(work.schedule())
    o = orc.FlashBlockOracle(spec.B, spec.Hq, spec.Hkv, spec.D, spec.Nb)
    kp, vp = work.prefix_kv()
    st = steps[2]
    o.step(orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin), orc.to64(kp), orc.to64(vp), st.prefix_len, 0, None,
           active=steps[2].active.numpy())
    with pytest.raises(AssertionError):   # a position locked at step 2 cannot be active again
        o.step(orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin), orc.to64(kp), orc.to64(vp), st.prefix_len, 0,
               None, active=steps[0].active.numpy())


# ------------------------------------------------ selection by attention mass ---
def test_attention_mass_sums_to_the_block_length_and_matches_brute_force():
    """Each query's probabilities over the prefix sum to 1, so a head's masses
    sum to Nb; on a tiny case every mass equals a 40-digit Decimal sum."""
    g = np.random.default_rng(3)
    Q = g.standard_normal((1, 2, 3, 4)); K = g.standard_normal((1, 1, 5, 4))
    M = orc.attention_mass(Q, K, 5, 0.7)
    np.testing.assert_allclose(M.sum(axis=2), 3.0, rtol=1e-14)
    decimal.getcontext().prec = 40
    for h in range(2):
        for j in range(5):
            tot = decimal.Decimal(0)
            for i in range(3):
                e = [(decimal.Decimal(0.7) * sum(decimal.Decimal(Q[0, h, i, d]) * decimal.Decimal(K[0, 0, jj, d])
                                                  for d in range(4))).exp() for jj in range(5)]
                tot += e[j] / sum(e)
            assert abs(float(tot) - M[0, h, j]) < 1e-14


def test_top_k_by_mass_closed_forms():
    # zero queries: every key gets mass Nb / n, all tied -> the first k keys
    Q = np.zeros((1, 1, 4, 8)); K = np.random.default_rng(4).standard_normal((1, 1, 10, 8))
    M = orc.attention_mass(Q, K, 10, 0.3)
    np.testing.assert_allclose(M, 0.4, rtol=1e-14)
    assert orc.select_top_k(M, 3).tolist() == [[[0, 1, 2]]]
    # a hand-worked ranking with a tie at the boundary: the lower index wins
    m = np.array([[[0.1, 0.5, 0.3, 0.5, 0.2, 0.3]]])
    assert orc.select_top_k(m, 3).tolist() == [[[1, 2, 3]]]
    assert orc.select_top_k(m, 4).tolist() == [[[1, 2, 3, 5]]]
    assert orc.select_top_k(m, 6).tolist() == [[[0, 1, 2, 3, 4, 5]]]
    # one dominant key per head (a key equal to a scaled query) ranks first
    K2 = np.zeros((1, 1, 6, 2)); K2[0, 0, 4] = [5.0, 0.0]
    Q2 = np.array([[[[1.0, 0.0]]]])
    assert orc.select_top_k(orc.attention_mass(Q2, K2, 6, 1.0), 1).tolist() == [[[4]]]


def test_static_queries_reuse_equals_full():
    """Queries unchanged across steps: the cached A_out is exact, so every step equals full attention."""
    spec, work = _tiny(steps=4)
    kp, vp = work.prefix_kv(); kp64, vp64 = orc.to64(kp), orc.to64(vp)
    o = orc.FlashBlockOracle(spec.B, spec.Hq, spec.Hkv, spec.D, spec.Nb)
    q0 = None
    for st in work.schedule():
        q0 = st.q if q0 is None else q0
        r = o.step(orc.to64(q0), orc.to64(st.kin), orc.to64(st.vin), kp64, vp64, st.prefix_len, 0, None)
        A, L = orc.full_attention(orc.to64(q0), orc.to64(st.kin), orc.to64(st.vin), kp64, vp64,
                                  st.prefix_len, 1 / 8)
        np.testing.assert_allclose(r.o, A, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(r.lse, L, rtol=1e-12)


def test_cosine_similarity_facts():
    rng = np.random.default_rng(7)
    a = rng.standard_normal(50); c = rng.standard_normal(50)
    assert orc.cosine_similarity(a, a) == pytest.approx(1.0, abs=1e-15)
    assert orc.cosine_similarity(a, -a) == pytest.approx(-1.0, abs=1e-15)
    assert orc.cosine_similarity(a, 3.5 * c) == pytest.approx(orc.cosine_similarity(a, c), abs=1e-15)
    e0 = np.eye(4)[0]; e1 = np.eye(4)[1]
    assert orc.cosine_similarity(e0, e1) == 0.0
    assert orc.cosine_similarity(e0 + e1, e0) == pytest.approx(1 / math.sqrt(2), abs=1e-15)
    assert orc.cosine_similarity(np.zeros(4), e0) == 0.0


def test_gamma_gate_per_head():
    """Head 0 never changes (sim 1 > gamma -> reuse from step 2); head 1 gets a
    new random query each step (sim well below gamma -> always recompute)."""
    rng = np.random.default_rng(8)
    B, H, Nb, D, Lp = 1, 2, 6, 8, 40
    kp = rng.standard_normal((B, H, Lp, D)); vp = rng.standard_normal((B, H, Lp, D))
    q = rng.standard_normal((B, H, Nb, D)); kin = rng.standard_normal((B, H, Nb, D))
    o = orc.FlashBlockOracle(B, H, H, D, Nb, gamma=[0.95, 0.95])
    o.begin_block()
    decisions = []
    for s in range(5):
        q = q.copy(); q[:, 1] = rng.standard_normal((B, Nb, D)) * 3
        r = o.step(q, kin, kin, kp, vp, Lp, Nb, None)
        decisions.append(r.head_reuse[0].tolist())
        if s >= 1:
            assert r.sim[0, 0] == pytest.approx(1.0, abs=1e-12)
            assert r.sim[0, 1] < 0.95
    assert decisions == [[False, False], [False, False], [True, False], [True, False], [True, False]]


def test_sparse_limits():
    """k = prefix: the residual set is empty, so a sparse step is a dense full
    step; k = 0: the selected set is empty, so the sparse step is dense FlashBlock."""
    spec, work = _tiny(steps=4)
    res_dense, _, _ = _run(spec, work, tau=spec.tau)
    kp, vp = work.prefix_kv(); kp64, vp64 = orc.to64(kp), orc.to64(vp)
    Lp = spec.prefix0
    all_sel = np.tile(np.arange(Lp, dtype=np.int32), (spec.B, spec.Hq, 1))
    no_sel = np.zeros((spec.B, spec.Hq, 0), dtype=np.int32)
    o_all = orc.FlashBlockOracle(spec.B, spec.Hq, spec.Hkv, spec.D, spec.Nb)
    o_none = orc.FlashBlockOracle(spec.B, spec.Hq, spec.Hkv, spec.D, spec.Nb)
    for (st, rd) in res_dense:
        args = (orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin), kp64, vp64, st.prefix_len, st.M, spec.tau)
        ra = o_all.step(*args, sel=all_sel)
        A, L = _full(st, kp64, vp64, 1 / 8)
        np.testing.assert_allclose(ra.o, A, rtol=1e-11, atol=1e-12)
        rn = o_none.step(*args, sel=no_sel)
        np.testing.assert_allclose(rn.o, rd.o, rtol=1e-12, atol=1e-13)
        assert rn.recompute == rd.recompute


def test_sparse_full_step_is_exact():
    spec, work = _tiny(steps=1)
    kp, vp = work.prefix_kv(); kp64, vp64 = orc.to64(kp), orc.to64(vp)
    rng = np.random.default_rng(9)
    sel = np.sort(np.stack([[rng.choice(spec.prefix0, 40, replace=False) for _ in range(spec.Hq)]]), axis=-1)
    st = next(work.schedule())
    o = orc.FlashBlockOracle(spec.B, spec.Hq, spec.Hkv, spec.D, spec.Nb)
    r = o.step(orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin), kp64, vp64, st.prefix_len, 0, 8, sel=sel)
    A, L = _full(st, kp64, vp64, 1 / 8)
    np.testing.assert_allclose(r.o, A, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(r.lse, L, rtol=1e-12)


def test_kv_append_positions():
    kp = np.zeros((1, 2, 10, 3)); vp = np.zeros((1, 2, 10, 3))
    kin = np.ones((1, 2, 4, 3)); vin = 2 * np.ones((1, 2, 4, 3))
    kp2, vp2, n = orc.kv_append(kp, vp, 5, kin, vin)
    assert n == 9
    assert np.all(kp2[:, :, 5:9] == 1) and np.all(kp2[:, :, :5] == 0) and np.all(kp2[:, :, 9:] == 0)
    assert np.all(vp2[:, :, 5:9] == 2)


# ----------------------------------------------- the pins have teeth ---
class _Planted:
    """A copy of the oracle module's namespace with one function replaced."""
    def __init__(self, **over):
        self.__dict__.update({k: getattr(orc, k) for k in dir(orc) if not k.startswith("__")})
        self.__dict__.update(over)


def _attn_transposed_v(q, k, v, scale):
    A, L = orc.attention_part(q, k, v, scale)
    s = scale * (np.asarray(q) @ np.asarray(k).T)
    e = np.exp(s - s.max(1, keepdims=True))
    return (e @ np.asarray(v)[::-1]) / e.sum(1, keepdims=True), L   # values in the wrong order


def _attn_no_scale(q, k, v, scale):
    return orc.attention_part(q, k, v, 1.0)


def _attn_lse_without_shift(q, k, v, scale):
    A, L = orc.attention_part(q, k, v, scale)
    s = scale * (np.asarray(q) @ np.asarray(k).T) if len(k) else np.zeros((len(q), 1))
    return A, L - s.max(1)                                             # dropped the max term


def _merge_wrong_sign(parts):
    flipped = [(a, -l) for a, l in parts]
    A, L = orc.merge(flipped)
    return A, -L


def _merge_unnormalised(parts):
    A, L = orc.merge(parts)
    m = np.max([l for _, l in parts], axis=0)
    return A, m                                                        # dropped log(sum w)


@pytest.mark.parametrize("planted, checks", [
    (dict(attention_part=_attn_transposed_v), ("brute", "golden")),
    (dict(attention_part=_attn_no_scale), ("brute", "golden", "softmax")),
    (dict(attention_part=_attn_lse_without_shift), ("brute", "golden", "softmax")),
    (dict(merge=_merge_wrong_sign), ("golden", "partition")),
    (dict(merge=_merge_unnormalised), ("golden", "partition")),
])
def test_planted_mistakes_are_caught(planted, checks):
    mod = _Planted(**planted)
    fns = {"brute": check_brute_force, "golden": check_golden, "closed": check_closed_forms,
           "softmax": check_softmax_special_case, "partition": check_partition_invariance}
    for name in checks:
        with pytest.raises(AssertionError):
            fns[name](mod)
