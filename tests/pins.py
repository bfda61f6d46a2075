"""Checks that pin the CPU oracle to facts other than itself.

Each pin_* function takes the path of an oracle build (None = the default
build) and raises AssertionError when the oracle disagrees with:
  * a two-step example worked out by hand (tests/golden/hand_two_steps.json);
  * brute force over all N slots for tiny N (the product-key identity
    topk(s1 (+) s2) = topk(topk(s1) (+) topk(s2)) of the SDM summaries,
    'Mecanismo Central' item 2);
  * special cases with closed forms: alpha=1, beta=0 leaves M bit-identical;
    beta*w = 1 overwrites the row with v_t exactly (and the read of the same
    step returns it); a single slot updated every step follows the geometric
    recurrence m_t = alpha(1-beta) m_{t-1} + beta v; softmax weight ratios equal
    exp(score differences); an all-zero query ties every score, so the lowest
    slots win; one-hot codebooks pin which half meets which codebook and the
    slot numbering i1*n + i2;
  * invariants: unselected rows stay bit-identical; splitting the time axis
    with the table carried over gives bit-identical results;
  * W = R = N (k = n): a dense all-slot gated delta update written with numpy;
  * the selective-decay write (the Raven page's rule on the same selection):
    a = 0 freezes every row, a very negative overwrites with v_t, a single slot
    follows e^{a t} m_0 + (1 - e^{a t}) v, router weights are normalised
    sigmoids, and one step from a known table moves only the selected rows;
  * the near-tie flags, from their definition in the workload specification (a
    float64 gap below 1e-5 relative at the W-th/(W+1)-th (R-th/(R+1)-th)
    candidate, or at a half's k-th/(k+1)-th row): hand-built score tables whose
    gaps are known by construction, just below and just above the threshold,
    for each bit.
The same functions are run against deliberately broken copies of the oracle
(tests/test_oracle_mutations.py) to show that each plausible mistake fails at
least one of them.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _dims(B=1, H=1, T=1, d_qk=8, d_v=4, n_sub=4, k=4, W=4, R=4):
    return dict(B=B, H=H, T=T, d_qk=d_qk, d_v=d_v, n_sub=n_sub, k=k, W=W, R=R)


def _rand_inputs(rng, d, m0_scale=0.0, alpha=None, beta=None):
    B, H, T = d['B'], d['H'], d['T']
    dh = d['d_qk'] // 2
    N = d['n_sub'] ** 2
    inp = dict(
        q=rng.standard_normal((B, H, T, d['d_qk'])).astype(np.float32),
        k=rng.standard_normal((B, H, T, d['d_qk'])).astype(np.float32),
        v=rng.standard_normal((B, H, T, d['d_v'])).astype(np.float32),
        alpha=(rng.uniform(0.5, 1.0, (B, H, T)) if alpha is None
               else np.full((B, H, T), alpha)).astype(np.float32),
        beta=(rng.uniform(0.0, 1.0, (B, H, T)) if beta is None
              else np.full((B, H, T), beta)).astype(np.float32),
        C1=(rng.standard_normal((H, d['n_sub'], dh)) / math.sqrt(dh)).astype(np.float32),
        C2=(rng.standard_normal((H, d['n_sub'], dh)) / math.sqrt(dh)).astype(np.float32),
        M0=(m0_scale * rng.standard_normal((B, H, N, d['d_v']))).astype(np.float32),
    )
    return inp


# ---------------------------------------------------------------- worked example
def pin_golden(so=None):
    with open(os.path.join(GOLDEN, "hand_two_steps.json")) as f:
        g = json.load(f)
    d = g['dims']
    inp = dict(q=np.array(g['q'], np.float32)[None, None], k=np.array(g['k'], np.float32)[None, None],
               v=np.array(g['v'], np.float32)[None, None],
               alpha=np.array(g['alpha'], np.float32)[None, None],
               beta=np.array(g['beta'], np.float32)[None, None],
               C1=np.array(g['C1'], np.float32)[None], C2=np.array(g['C2'], np.float32)[None],
               M0=np.array(g['M0'], np.float32)[None, None])
    out = oracle.forward(inp, d, lists=True, so=so)
    e = g['expect']
    assert out['idx_w'][0, 0].tolist() == e['idx_w'], out['idx_w'][0, 0]
    assert out['idx_r'][0, 0].tolist() == e['idx_r'], out['idx_r'][0, 0]
    np.testing.assert_allclose(out['w_w'][0, 0], np.array(e['w_w']), rtol=1e-12)
    np.testing.assert_allclose(out['o'][0, 0], np.array(e['o']), rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(out['M'][0, 0], np.array(e['M']), rtol=1e-6, atol=1e-7)


# ---------------------------------------------------------------- brute force over N
def _brute_topk(x, C1, C2, n, n_sel):
    """All N = n^2 slot scores materialised; order (score desc, slot asc)."""
    dh = x.shape[0] // 2
    s1 = (C1.astype(np.float64) @ x[:dh].astype(np.float64)).astype(np.float32)
    s2 = (C2.astype(np.float64) @ x[dh:].astype(np.float64)).astype(np.float32)
    S = (s1[:, None] + s2[None, :]).reshape(-1)       # float32 sums, slot = i1*n + i2
    slots = np.arange(n * n)
    order = np.lexsort((slots, -S.astype(np.float64)))
    top = order[:n_sel]
    sel = S[top].astype(np.float64)
    w = np.exp(sel - sel.max())
    return top, w / w.sum()


def pin_bruteforce_identity(so=None):
    rng = np.random.default_rng(1234)
    for trial in range(60):
        n = int(rng.choice([4, 6, 8, 16]))
        dh = int(rng.choice([1, 2, 4, 8]))
        k = int(rng.integers(1, n + 1))
        n_sel = int(rng.integers(1, k + 1))            # k >= n_sel: the identity is exact
        d = _dims(d_qk=2 * dh, n_sub=n, k=k, W=n_sel, R=n_sel)
        x = rng.standard_normal(2 * dh).astype(np.float32)
        C1 = rng.standard_normal((n, dh)).astype(np.float32)
        C2 = rng.standard_normal((n, dh)).astype(np.float32)
        if trial % 3 == 0:                             # adversarial exact ties
            C1[1::2] = C1[0::2][: C1[1::2].shape[0]]
            C2[2] = C2[0]
        if trial % 5 == 0:
            x[:dh] = 0.0
        slots, w, _, _ = oracle.select(x, C1, C2, d, n_sel, so=so)
        top, wb = _brute_topk(x, C1, C2, n, n_sel)
        assert slots.tolist() == top.tolist(), (trial, slots, top)
        np.testing.assert_allclose(w, wb, rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- closed forms
def pin_gates_identity(so=None):
    """alpha = 1, beta = 0: (1-0)*(1*M) + 0*v = M, every row bit-identical."""
    rng = np.random.default_rng(7)
    d = _dims(B=2, H=2, T=40, d_qk=8, d_v=6, n_sub=5, k=3, W=4, R=5)
    inp = _rand_inputs(rng, d, m0_scale=1.0, alpha=1.0, beta=0.0)
    out = oracle.forward(inp, d, so=so)
    assert np.array_equal(out['M'], inp['M0'])


def pin_overwrite_and_read_after_write(so=None):
    """W = R = 1 (weights exactly 1), beta = 1 and q' = k': the written row becomes
    v_t exactly and the read of the same step returns v_t."""
    rng = np.random.default_rng(8)
    d = _dims(B=1, H=2, T=30, d_qk=6, d_v=5, n_sub=6, k=2, W=1, R=1)
    inp = _rand_inputs(rng, d, m0_scale=1.0, beta=1.0)
    inp['q'] = inp['k'].copy()
    out = oracle.forward(inp, d, lists=True, so=so)
    assert np.array_equal(out['o'], inp['v'])
    for h in range(2):
        for t in range(d['T']):
            s = int(out['idx_w'][0, h, t, 0])
            last = max(u for u in range(d['T']) if int(out['idx_w'][0, h, u, 0]) == s)
            assert np.array_equal(out['M'][0, h, s], inp['v'][0, h, last])


def pin_single_slot_recurrence(so=None):
    """One slot wins every step (W = R = 1, constant alpha, beta, v):
    m_t = a m_{t-1} + beta v with a = alpha (1 - beta), so
    m_T = a^T m_0 + beta v (1 - a^T) / (1 - a); and o_t = m_t."""
    n, dh, T = 4, 4, 50
    d = _dims(T=T, d_qk=2 * dh, d_v=3, n_sub=n, k=2, W=1, R=1)
    rng = np.random.default_rng(9)
    C1 = 0.01 * rng.standard_normal((1, n, dh)).astype(np.float32)
    C2 = 0.01 * rng.standard_normal((1, n, dh)).astype(np.float32)
    C1[0, 2] = 5.0
    C2[0, 1] = 5.0
    keys = (np.abs(rng.standard_normal((1, 1, T, 2 * dh))) + 0.5).astype(np.float32)
    al, be = 0.9, 0.3
    vv = np.array([1.0, -2.0, 0.5], np.float32)
    m0 = np.zeros((1, 1, n * n, 3), np.float32)
    m0[0, 0, 2 * n + 1] = [4.0, 4.0, -4.0]
    inp = dict(q=keys.copy(), k=keys, v=np.broadcast_to(vv, (1, 1, T, 3)).copy(),
               alpha=np.full((1, 1, T), al, np.float32), beta=np.full((1, 1, T), be, np.float32),
               C1=C1, C2=C2, M0=m0)
    out = oracle.forward(inp, d, lists=True, so=so)
    assert (out['idx_w'][0, 0, :, 0] == 2 * n + 1).all()
    a = float(np.float32(al)) * (1.0 - float(np.float32(be)))
    b = float(np.float32(be))
    tt = np.arange(1, T + 1)[:, None]
    expect = a ** tt * m0[0, 0, 2 * n + 1][None, :] + b * vv[None, :] * (1 - a ** tt) / (1 - a)
    np.testing.assert_allclose(out['o'][0, 0], expect, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(out['M'][0, 0, 2 * n + 1], expect[-1], rtol=1e-5, atol=1e-6)


def pin_softmax_weights(so=None):
    """w_i / w_j = exp(s_i - s_j) over the selected float32 scores; sum 1;
    non-increasing along the rank order."""
    rng = np.random.default_rng(10)
    for _ in range(20):
        d = _dims(d_qk=8, n_sub=8, k=4, W=6, R=6)
        x = rng.standard_normal(8).astype(np.float32) * 3
        C1 = rng.standard_normal((8, 4)).astype(np.float32)
        C2 = rng.standard_normal((8, 4)).astype(np.float32)
        slots, w, s, _ = oracle.select(x, C1, C2, d, 6, so=so)
        assert abs(w.sum() - 1.0) < 1e-12
        assert (np.diff(s.astype(np.float64)) <= 0).all()
        ratio = w[:, None] / w[None, :]
        expect = np.exp(s.astype(np.float64)[:, None] - s.astype(np.float64)[None, :])
        np.testing.assert_allclose(ratio, expect, rtol=1e-12)


def pin_ties_lowest_index(so=None):
    """x = 0: every half score is 0, every candidate ties; the lower index wins
    in each half (ranks 0..k-1 are codebook rows 0..k-1) and among slots, so the
    selection is slots 0..n_sel-1 (i1 = 0, i2 = 0..n_sel-1) with uniform weights."""
    for n, k, n_sel in [(8, 4, 3), (6, 6, 6), (10, 7, 5)]:
        d = _dims(d_qk=6, n_sub=n, k=k, W=n_sel, R=n_sel)
        rng = np.random.default_rng(n)
        C1 = rng.standard_normal((n, 3)).astype(np.float32)
        C2 = rng.standard_normal((n, 3)).astype(np.float32)
        slots, w, _, _ = oracle.select(np.zeros(6, np.float32), C1, C2, d, n_sel, so=so)
        assert slots.tolist() == list(range(n_sel)), slots
        np.testing.assert_allclose(w, np.full(n_sel, 1.0 / n_sel), rtol=1e-14)


def pin_half_split_and_slot_numbering(so=None):
    """One-hot codebooks: the first half of x meets C1, the second half C2, and
    the winning slot is i1 * n + i2."""
    n, dh = 8, 8
    d = _dims(d_qk=2 * dh, n_sub=n, k=2, W=1, R=1)
    C1 = np.eye(n, dh, dtype=np.float32)
    C2 = np.eye(n, dh, dtype=np.float32)
    for i1, i2 in [(3, 1), (6, 2), (0, 7)]:
        x = np.zeros(2 * dh, np.float32)
        x[i1] = 1.0
        x[dh + i2] = 1.0
        slots, _, s, _ = oracle.select(x, C1, C2, d, 1, so=so)
        assert int(slots[0]) == i1 * n + i2, (slots, i1, i2)
        assert float(s[0]) == 2.0


# ---------------------------------------------------------------- invariants
def pin_untouched_rows(so=None):
    rng = np.random.default_rng(11)
    d = _dims(B=1, H=3, T=25, d_qk=8, d_v=4, n_sub=6, k=3, W=4, R=3)
    inp = _rand_inputs(rng, d, m0_scale=1.0)
    out = oracle.forward(inp, d, lists=True, so=so)
    for h in range(3):
        written = set(out['idx_w'][0, h].reshape(-1).tolist())
        other = np.array(sorted(set(range(36)) - written), dtype=np.int64)
        assert np.array_equal(out['M'][0, h, other], inp['M0'][0, h, other])
        assert not np.array_equal(out['M'][0, h, sorted(written)], inp['M0'][0, h, sorted(written)])


def pin_streaming(so=None):
    rng = np.random.default_rng(12)
    d = _dims(B=2, H=2, T=33, d_qk=8, d_v=4, n_sub=5, k=4, W=5, R=3)
    inp = _rand_inputs(rng, d, m0_scale=0.5)
    full = oracle.forward(inp, d, so=so)
    M = inp['M0'].copy()
    a = oracle.forward(inp, d, t_begin=0, t_end=14, M=M, so=so)
    b = oracle.forward(inp, d, t_begin=14, t_end=33, M=M, so=so)
    assert np.array_equal(M, full['M'])
    o = np.concatenate([a['o'][:, :, :14], b['o'][:, :, 14:]], axis=2)
    assert np.array_equal(o, full['o'])


def _dense_reference(inp, d):
    """W = R = N with k = n: every slot is selected; all-slot softmax weights."""
    n = d['n_sub']
    dh = d['d_qk'] // 2
    B, H, T = d['B'], d['H'], d['T']
    M = inp['M0'].astype(np.float32).copy()
    o = np.zeros((B, H, T, d['d_v']), np.float32)
    for b in range(B):
        for h in range(H):
            C1 = inp['C1'][h].astype(np.float64)
            C2 = inp['C2'][h].astype(np.float64)

            def scores(x):
                s1 = (C1 @ x[:dh].astype(np.float64)).astype(np.float32)
                s2 = (C2 @ x[dh:].astype(np.float64)).astype(np.float32)
                return (s1[:, None] + s2[None, :]).reshape(-1).astype(np.float64)

            for t in range(T):
                sw = scores(inp['k'][b, h, t])
                w = np.exp(sw - sw.max())
                w /= w.sum()
                c = float(inp['beta'][b, h, t]) * w
                mt = float(inp['alpha'][b, h, t]) * M[b, h].astype(np.float64)
                M[b, h] = ((1.0 - c)[:, None] * mt
                           + c[:, None] * inp['v'][b, h, t].astype(np.float64)[None, :]).astype(np.float32)
                sr = scores(inp['q'][b, h, t])
                u = np.exp(sr - sr.max())
                u /= u.sum()
                o[b, h, t] = (u @ M[b, h].astype(np.float64)).astype(np.float32)
    return o, M


def pin_dense_all_slots(so=None):
    rng = np.random.default_rng(13)
    n = 4
    d = _dims(B=1, H=2, T=20, d_qk=6, d_v=3, n_sub=n, k=n, W=n * n, R=n * n)
    inp = _rand_inputs(rng, d, m0_scale=1.0)
    out = oracle.forward(inp, d, so=so)
    o, M = _dense_reference(inp, d)
    np.testing.assert_allclose(out['M'], M, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(out['o'], o, rtol=1e-6, atol=1e-6)


# ---------------------------------------------------------------- near-tie flags
# Score tables with n = 4 rows per half, k = 2, W = R = 2.  The key k' uses
# coordinate 0 of each half and the query q' coordinate 1 (d_h = 2), so
# C1[:, 0] / C2[:, 0] are the key's half-score tables and C1[:, 1] / C2[:, 1]
# the query's, and each side's flags can be driven on its own.
#
# base: s1 = [3, 2, 0, -1], s2 = [3, 1, 0, -1].  Candidates of the top-2 rows:
#   6, 5, 4, 3 -> the 2nd/3rd gap is 1/5; each half's rank-1/rank-2 gap is large.
_FLAG_BASE = ([3.0, 2.0, 0.0, -1.0], [3.0, 1.0, 0.0, -1.0])


def _flag_tables(case, delta):
    """(s1, s2) of a side whose relative gap `delta` sits where `case` says:
    'boundary': the 2nd/3rd candidate, 5 and 5 - 5 delta (bit 0 / 3);
    'half1'   : half 1's k-th/(k+1)-th rows, 2 and 2 - 2 delta (bit 1 / 4);
    'half2'   : half 2's k-th/(k+1)-th rows, 1 and 1 - delta (bit 2 / 5);
    'rank01'  : half 1's 1st/2nd rows, 3 and 3 - 3 delta, which are not at
                any selection boundary (no bit)."""
    s1, s2 = list(_FLAG_BASE[0]), list(_FLAG_BASE[1])
    if case == "boundary":
        s2[1] = 2.0 - 5.0 * delta     # candidates 6, 5, 5 - 5 delta, 4 - 5 delta
    elif case == "half1":
        s1[2] = 2.0 - 2.0 * delta
    elif case == "half2":
        s2[2] = 1.0 - delta
    elif case == "rank01":
        s1[1] = 3.0 - 3.0 * delta     # candidates 6, 6 - 3 delta, 4, ...: 2nd/3rd far
    return s1, s2


_FLAG_BIT = {"boundary": 1, "half1": 2, "half2": 4, "rank01": 0}


def pin_near_tie_flags(so=None):
    d = _dims(T=1, d_qk=4, d_v=4, n_sub=4, k=2, W=2, R=2)
    for side in ("key", "query"):
        for case in ("boundary", "half1", "half2", "rank01"):
            for delta, flagged in ((0.9e-5, True), (1.1e-5, False)):
                t1, t2 = _flag_tables(case, delta)
                b1, b2 = _FLAG_BASE
                key1, key2 = (t1, t2) if side == "key" else (b1, b2)
                qry1, qry2 = (t1, t2) if side == "query" else (b1, b2)
                C1 = np.array([key1, qry1], np.float32).T[None]      # [1, n, 2]
                C2 = np.array([key2, qry2], np.float32).T[None]
                inp = dict(k=np.array([1, 0, 1, 0], np.float32)[None, None, None],
                           q=np.array([0, 1, 0, 1], np.float32)[None, None, None],
                           v=np.ones((1, 1, 1, 4), np.float32),
                           alpha=np.ones((1, 1, 1), np.float32),
                           beta=np.ones((1, 1, 1), np.float32), C1=C1, C2=C2,
                           M0=np.zeros((1, 1, 16, 4), np.float32))
                out = oracle.forward(inp, d, lists=True, so=so)
                bit = _FLAG_BIT[case] if flagged else 0
                expect = bit if side == "key" else bit << 3
                got = int(out['flags'][0, 0, 0])
                assert got == expect, (side, case, delta, got, expect)


def pin_near_tie_flags_float64_gap(so=None):
    """The flag reads the float64 gap, not the float32 one.  s1 = [1, 1 - g, -10],
    s2 = [2^-24, -10, -20], x = [1, 1], W = 1, k = 2, g = 168 * 2^-24.  The best
    candidate is 1 + 2^-24 exactly in float64, which rounds (to even) to 1.0 in
    float32; the second is 1 - 167 * 2^-24 exactly in both.  The float64 gap,
    168 * 2^-24 / (1 + 2^-24) = 1.0014e-5 relative, is above 1e-5 (no flag); the
    float32 one, 167 * 2^-24 = 9.95e-6, would be below it."""
    e = 2.0 ** -24
    g = 168 * e
    d = _dims(d_qk=2, n_sub=3, k=2, W=1, R=1)
    C1 = np.array([[1.0], [1.0 - g], [-10.0]], np.float32)
    C2 = np.array([[e], [-10.0], [-20.0]], np.float32)
    assert float(C1[1, 0]) == 1.0 - g and float(C2[0, 0]) == e
    assert np.float32(1.0) + np.float32(e) == np.float32(1.0)
    slots, _, s, flag = oracle.select(np.array([1.0, 1.0], np.float32), C1, C2, d, 1, so=so)
    assert int(slots[0]) == 0 and float(s[0]) == 1.0
    assert flag == 0, flag
    # the same tables with g = 167 * 2^-24: the float64 gap is below 1e-5
    C1[1, 0] = np.float32(1.0 - 167 * e)
    _, _, _, flag = oracle.select(np.array([1.0, 1.0], np.float32), C1, C2, d, 1, so=so)
    assert flag == 1, flag


# ---------------------------------------------------------------- selective decay
# The Raven page's write rule on the product-key selection (oracle.forward_decay):
# r = sigmoid(score) normalised over the W selected slots; M[i] = exp(a r_i) M[i]
# + (1 - exp(a r_i)) v_t on the selected rows only.
def _decay_inp(rng, d, a):
    inp = _rand_inputs(rng, d, m0_scale=1.0)
    inp['a'] = (np.full(inp['alpha'].shape, a) if np.isscalar(a) else a).astype(np.float32)
    return inp


def pin_decay_frozen_and_overwrite(so=None):
    """a = 0: exp(0) = 1, every row frozen (bit-identical).  a = -1e4 with W = R = 1
    (r = 1, exp(-1e4) = 0 in float64) and q' = k': the written row becomes v_t
    exactly and the same step's read returns it."""
    rng = np.random.default_rng(31)
    d = _dims(B=1, H=2, T=30, d_qk=8, d_v=4, n_sub=5, k=3, W=4, R=3)
    inp = _decay_inp(rng, d, 0.0)
    out = oracle.forward_decay(inp, d, so=so)
    assert np.array_equal(out['M'], inp['M0'])
    d1 = _dims(B=1, H=2, T=30, d_qk=6, d_v=5, n_sub=6, k=2, W=1, R=1)
    inp = _decay_inp(rng, d1, -1e4)
    inp['q'] = inp['k'].copy()
    out = oracle.forward_decay(inp, d1, so=so)
    assert np.array_equal(out['o'], inp['v'])


def pin_decay_single_slot(so=None):
    """One slot wins every step (W = R = 1, r = 1): m_t = e^a m_{t-1} + (1 - e^a) v,
    so m_t = e^{a t} m_0 + (1 - e^{a t}) v and o_t = m_t."""
    n, dh, T = 4, 4, 40
    d = _dims(T=T, d_qk=2 * dh, d_v=3, n_sub=n, k=2, W=1, R=1)
    rng = np.random.default_rng(32)
    C1 = 0.01 * rng.standard_normal((1, n, dh)).astype(np.float32)
    C2 = 0.01 * rng.standard_normal((1, n, dh)).astype(np.float32)
    C1[0, 1] = 5.0
    C2[0, 3] = 5.0
    keys = (np.abs(rng.standard_normal((1, 1, T, 2 * dh))) + 0.5).astype(np.float32)
    vv = np.array([2.0, -1.0, 0.25], np.float32)
    m0 = np.zeros((1, 1, n * n, 3), np.float32)
    m0[0, 0, 1 * n + 3] = [1.0, 1.0, 1.0]
    a = np.float32(-0.3)
    inp = dict(q=keys.copy(), k=keys, v=np.broadcast_to(vv, (1, 1, T, 3)).copy(),
               a=np.full((1, 1, T), a, np.float32), C1=C1, C2=C2, M0=m0)
    out = oracle.forward_decay(inp, d, lists=True, so=so)
    assert (out['idx_w'][0, 0, :, 0] == 1 * n + 3).all()
    assert (out['w_w'][0, 0, :, 0] == 1.0).all()
    e = np.exp(float(a) * np.arange(1, T + 1))[:, None]
    expect = e * m0[0, 0, 1 * n + 3][None, :] + (1.0 - e) * vv[None, :].astype(np.float64)
    np.testing.assert_allclose(out['o'][0, 0], expect, rtol=1e-5, atol=1e-6)


def pin_decay_router_weights(so=None):
    """r_i / r_j = sigmoid(s_i) / sigmoid(s_j) over the selected float32 scores, sum
    1; the selection itself is the product-key top-W (same slots as the oracle's
    selection of that key)."""
    rng = np.random.default_rng(33)
    d = _dims(B=1, H=1, T=12, d_qk=8, d_v=4, n_sub=8, k=4, W=6, R=6)
    inp = _decay_inp(rng, d, -0.5)
    out = oracle.forward_decay(inp, d, lists=True, so=so)
    for t in range(12):
        slots, _, s, _ = oracle.select(inp['k'][0, 0, t], inp['C1'][0], inp['C2'][0], d, 6, so=so)
        assert out['idx_w'][0, 0, t].tolist() == slots.tolist()
        sig = 1.0 / (1.0 + np.exp(-s.astype(np.float64)))
        np.testing.assert_allclose(out['w_w'][0, 0, t], sig / sig.sum(), rtol=1e-12)


def pin_decay_one_step_rows(so=None):
    """One step from a known table: each selected row i becomes
    exp(a r_i) M0[i] + (1 - exp(a r_i)) v; every other row is unchanged."""
    rng = np.random.default_rng(34)
    d = _dims(B=1, H=1, T=1, d_qk=8, d_v=4, n_sub=6, k=3, W=5, R=2)
    inp = _decay_inp(rng, d, -0.8)
    out = oracle.forward_decay(inp, d, lists=True, so=so)
    M0 = inp['M0'][0, 0].astype(np.float64)
    sel = out['idx_w'][0, 0, 0]
    r = out['w_w'][0, 0, 0]
    expect = M0.copy()
    for i, ri in zip(sel, r):
        dcy = np.exp(-0.8 * ri)
        expect[i] = dcy * M0[i] + (1.0 - dcy) * inp['v'][0, 0, 0].astype(np.float64)
    np.testing.assert_allclose(out['M'][0, 0], expect, rtol=1e-6, atol=1e-7)
    other = np.setdiff1d(np.arange(36), sel)
    assert np.array_equal(out['M'][0, 0, other], inp['M0'][0, 0, other])


ALL_PINS = [pin_golden, pin_bruteforce_identity, pin_gates_identity,
            pin_overwrite_and_read_after_write, pin_single_slot_recurrence, pin_softmax_weights,
            pin_ties_lowest_index, pin_half_split_and_slot_numbering, pin_untouched_rows,
            pin_streaming, pin_dense_all_slots, pin_near_tie_flags,
            pin_near_tie_flags_float64_gap, pin_decay_frozen_and_overwrite, pin_decay_single_slot,
            pin_decay_router_weights, pin_decay_one_step_rows]
