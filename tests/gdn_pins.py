"""Checks that pin the dense GDN oracle (oracle/gdn_oracle.c) to facts other
than itself.  Each pin takes the path of an oracle build (None = default) and
raises AssertionError on disagreement with:
  * the expanded matrix form of the rule, S_t = alpha_t S_{t-1} (I - beta_t
    k_t k_t^T) + beta_t v_t k_t^T, multiplied out with numpy matrices (the
    oracle evaluates the residual form row by row);
  * one-hot keys and queries (k_t = e_j, q_t = e_l): column j follows the
    scalar gated delta update alpha (1 - beta) s + beta v, the other columns
    decay by alpha, and o_t is column l -- the hard single-slot case of the
    SDM update;
  * alpha = 1, beta = 0: S never changes and o_t = S_0 q_t;
  * alpha = 1, beta = 1 and unit-norm keys: after each step S_t k_t = v_t
    (the delta rule's exact recall), so with q_t = k_t the read returns v_t;
  * beta = 0: S_t = alpha^t S_0 (pure decay);
  * splitting the sequence with the state carried (as float32) between calls.
"""
from __future__ import annotations

import numpy as np

import oracle


def _inp(rng, B, H, T, dk, dv, s0=1.0):
    return dict(q=rng.standard_normal((B, H, T, dk)).astype(np.float32),
                k=(rng.standard_normal((B, H, T, dk)) / np.sqrt(dk)).astype(np.float32),
                v=rng.standard_normal((B, H, T, dv)).astype(np.float32),
                alpha=rng.uniform(0.6, 1.0, (B, H, T)).astype(np.float32),
                beta=rng.uniform(0.0, 1.0, (B, H, T)).astype(np.float32),
                S0=(s0 * rng.standard_normal((B, H, dv, dk))).astype(np.float32))


def _dims(inp):
    B, H, T, dk = inp['q'].shape
    return dict(B=B, H=H, T=T, d_k=dk, d_v=inp['v'].shape[-1])


def pin_gdn_matrix_form(so=None):
    rng = np.random.default_rng(21)
    inp = _inp(rng, 2, 2, 30, 5, 3)
    out = oracle.gdn_forward(inp, _dims(inp), so=so)
    for b in range(2):
        for h in range(2):
            S = inp['S0'][b, h].astype(np.float64)
            for t in range(30):
                k = inp['k'][b, h, t].astype(np.float64)
                v = inp['v'][b, h, t].astype(np.float64)
                a, be = float(inp['alpha'][b, h, t]), float(inp['beta'][b, h, t])
                S = a * S @ (np.eye(5) - be * np.outer(k, k)) + be * np.outer(v, k)
                o = S @ inp['q'][b, h, t].astype(np.float64)
                np.testing.assert_allclose(out['o'][b, h, t], o, rtol=1e-5, atol=1e-6)
            np.testing.assert_allclose(out['S'][b, h], S, rtol=1e-5, atol=1e-6)


def pin_gdn_one_hot(so=None):
    rng = np.random.default_rng(22)
    B, H, T, dk, dv = 1, 2, 40, 6, 4
    inp = _inp(rng, B, H, T, dk, dv)
    js = rng.integers(0, dk, (B, H, T))
    ls = rng.integers(0, dk, (B, H, T))
    inp['k'] = np.eye(dk, dtype=np.float32)[js]
    inp['q'] = np.eye(dk, dtype=np.float32)[ls]
    out = oracle.gdn_forward(inp, _dims(inp), so=so)
    for h in range(H):
        S = inp['S0'][0, h].astype(np.float64)
        for t in range(T):
            a, be = float(inp['alpha'][0, h, t]), float(inp['beta'][0, h, t])
            j = js[0, h, t]
            col = a * (1.0 - be) * S[:, j] + be * inp['v'][0, h, t].astype(np.float64)
            S = a * S
            S[:, j] = col
            np.testing.assert_allclose(out['o'][0, h, t], S[:, ls[0, h, t]], rtol=1e-6,
                                       atol=1e-7)
        np.testing.assert_allclose(out['S'][0, h], S, rtol=1e-6, atol=1e-7)


def pin_gdn_gates_identity(so=None):
    rng = np.random.default_rng(23)
    inp = _inp(rng, 1, 2, 25, 4, 5)
    inp['alpha'][:] = 1.0
    inp['beta'][:] = 0.0
    out = oracle.gdn_forward(inp, _dims(inp), so=so)
    assert np.array_equal(out['S'], inp['S0'])
    o = np.einsum('bhvk,bhtk->bhtv', inp['S0'].astype(np.float64), inp['q'].astype(np.float64))
    np.testing.assert_allclose(out['o'], o, rtol=1e-6, atol=1e-7)


def pin_gdn_exact_recall(so=None):
    rng = np.random.default_rng(24)
    inp = _inp(rng, 1, 2, 30, 8, 3)
    k = inp['k'].astype(np.float64)
    inp['k'] = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
    inp['q'] = inp['k'].copy()
    inp['alpha'][:] = 1.0
    inp['beta'][:] = 1.0
    out = oracle.gdn_forward(inp, _dims(inp), so=so)
    # |k|^2 is 1 up to float32 rounding of k
    np.testing.assert_allclose(out['o'], inp['v'], rtol=1e-5, atol=1e-5)


def pin_gdn_pure_decay(so=None):
    rng = np.random.default_rng(25)
    inp = _inp(rng, 1, 1, 20, 4, 4)
    inp['beta'][:] = 0.0
    inp['alpha'][:] = np.float32(0.9)
    out = oracle.gdn_forward(inp, _dims(inp), so=so)
    a = float(np.float32(0.9))
    S0 = inp['S0'][0, 0].astype(np.float64)
    for t in range(20):
        o = a ** (t + 1) * S0 @ inp['q'][0, 0, t].astype(np.float64)
        np.testing.assert_allclose(out['o'][0, 0, t], o, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(out['S'][0, 0], a ** 20 * S0, rtol=1e-6, atol=1e-7)


def pin_gdn_streaming(so=None):
    rng = np.random.default_rng(26)
    inp = _inp(rng, 2, 1, 33, 5, 4)
    d = _dims(inp)
    full = oracle.gdn_forward(inp, d, so=so)
    S = inp['S0'].copy()
    a = oracle.gdn_forward(inp, d, t_end=12, S=S, so=so)
    b = oracle.gdn_forward(inp, d, t_begin=12, S=S, so=so)
    o = np.concatenate([a['o'][:, :, :12], b['o'][:, :, 12:]], axis=2)
    # the state crosses the split as float32: agreement to float32 rounding
    np.testing.assert_allclose(o, full['o'], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(S, full['S'], rtol=1e-5, atol=1e-6)


GDN_PINS = [pin_gdn_matrix_form, pin_gdn_one_hot, pin_gdn_gates_identity, pin_gdn_exact_recall,
            pin_gdn_pure_decay, pin_gdn_streaming]
