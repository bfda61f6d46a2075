"""The reference gradients (oracle/backward.py) against things other than
themselves: its float64 forward reproduces the C oracle's o and M_T (to float32
rounding, at the C oracle's selections); its gradients equal central finite
differences of that forward for every input on small problems; and one slot
written and read every step has closed-form gradients."""
import numpy as np
import pytest

import oracle
from oracle import backward as ob
from pins import _dims, _rand_inputs


def _case(seed, **kw):
    rng = np.random.default_rng(seed)
    d = _dims(**kw)
    inp = _rand_inputs(rng, d, m0_scale=1.0)
    out = oracle.forward(inp, d, lists=True)
    return rng, d, inp, out


def test_forward64_matches_the_c_oracle():
    _, d, inp, out = _case(41, B=1, H=2, T=30, d_qk=8, d_v=5, n_sub=6, k=4, W=5, R=3)
    x = {nm: ob._t64(inp[nm]) for nm in ob.NAMES}
    o, M = ob.forward64(x, out, d)
    np.testing.assert_allclose(o.numpy(), out['o'], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(M.numpy(), out['M'], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("seed,shape", [
    (42, dict(B=1, H=1, T=6, d_qk=4, d_v=3, n_sub=4, k=3, W=3, R=2)),
    (43, dict(B=1, H=2, T=5, d_qk=6, d_v=2, n_sub=5, k=2, W=2, R=4)),
])
def test_gradients_match_finite_differences(seed, shape):
    rng, d, inp, out = _case(seed, **shape)
    do = rng.standard_normal(out['o'].shape)
    dM = rng.standard_normal(out['M'].shape)
    g = ob.grads(inp, out, d, do, dM)
    h = 1e-6
    for nm in ob.NAMES:
        a = inp[nm].astype(np.float64)
        flat = a.reshape(-1)
        # every element of the small tensors, a sample of the table's
        idx = range(flat.size) if flat.size <= 200 else rng.choice(flat.size, 200, replace=False)
        for i in idx:
            old = flat[i]
            flat[i] = old + h
            lp = ob.loss64(dict(inp, **{nm: a}), out, d, do, dM)
            flat[i] = old - h
            lm = ob.loss64(dict(inp, **{nm: a}), out, d, do, dM)
            flat[i] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g[nm].reshape(-1)[i]) <= 1e-6 * max(1.0, abs(fd)), (nm, i, fd,
                                                                                g[nm].reshape(-1)[i])


def test_single_slot_closed_form():
    """W = R = 1, one slot every step, constant alpha, beta: m_t = a m_{t-1} + beta v_t
    with a = alpha (1 - beta), o_t = m_t (w = u = 1, so the scores get no
    gradient).  With L = sum_t o_t . g_t: dL/dv_s = beta sum_{t>=s} a^{t-s} g_t and
    dL/dm_0 = sum_t a^t g_t (t counted from 1)."""
    n, dh, T = 4, 4, 12
    d = _dims(T=T, d_qk=2 * dh, d_v=2, n_sub=n, k=2, W=1, R=1)
    rng = np.random.default_rng(44)
    C1 = 0.01 * rng.standard_normal((1, n, dh)).astype(np.float32)
    C2 = 0.01 * rng.standard_normal((1, n, dh)).astype(np.float32)
    C1[0, 2] = 5.0
    C2[0, 1] = 5.0
    keys = (np.abs(rng.standard_normal((1, 1, T, 2 * dh))) + 0.5).astype(np.float32)
    al, be = np.float32(0.9), np.float32(0.3)
    inp = dict(q=keys.copy(), k=keys, v=rng.standard_normal((1, 1, T, 2)).astype(np.float32),
               alpha=np.full((1, 1, T), al, np.float32), beta=np.full((1, 1, T), be, np.float32),
               C1=C1, C2=C2, M0=rng.standard_normal((1, 1, n * n, 2)).astype(np.float32))
    out = oracle.forward(inp, d, lists=True)
    slot = 2 * n + 1
    assert (out['idx_w'] == slot).all() and (out['idx_r'] == slot).all()
    gt = rng.standard_normal((1, 1, T, 2))
    g = ob.grads(inp, out, d, gt)
    a = float(al) * (1.0 - float(be))
    for s in range(T):
        expect = float(be) * sum(a ** (t - s) * gt[0, 0, t] for t in range(s, T))
        np.testing.assert_allclose(g['v'][0, 0, s], expect, rtol=1e-10)
    np.testing.assert_allclose(g['M0'][0, 0, slot], sum(a ** (t + 1) * gt[0, 0, t]
                                                        for t in range(T)), rtol=1e-10)
    assert np.abs(g['C1']).max() < 1e-12 and np.abs(g['q']).max() < 1e-12
