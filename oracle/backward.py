"""Reference gradients of the SDM forward pass -- TEST INFRASTRUCTURE ONLY.

Only tests/ may import this module; the product path never does.

What it computes.  The SDM summaries (gist.science 2607.07386) train the whole
model, the initial table M_0 included ("Estado Inicial Aprendido": M_0 is a
learned parameter), but give no backward pass.  The gradient of the method is
taken here as the derivative of the forward pass ("Mecanismo Central" items
2-4) with the discrete choices -- each half's top-k and the top-W / top-R
candidates -- held at the ones the forward pass made (they are piecewise
constant in the inputs, so this is the derivative wherever no near-tie sits at
a selection boundary).  Through those fixed choices the scores are real-valued:

    s1[j] = x[0:d_h] . C1[j],   s2[j] = x[d_h:] . C2[j]      (x = k'_t or q'_t)
    score(i1 * n + i2) = s1[i1] + s2[i2]
    w = softmax of the W write scores, u = softmax of the R read scores
    M~[i] = alpha_t M[i];  M[i] = M~[i] + beta_t w_i (v_t - M~[i])   (write slots)
    o_t = sum_r u_r M_t[r]                                            (after the write)

The forward is written out with plain float64 torch operations (no rounding to
float32 anywhere) and differentiated by torch.autograd, a library primitive.
Its values agree with the C oracle's to float32 rounding (a test checks this),
and its gradients agree with central finite differences of the same forward on
small problems (a test checks this too).
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch


def _t64(a, grad=False):
    t = torch.as_tensor(np.asarray(a, dtype=np.float64))
    return t.requires_grad_(grad)


def forward64(x: Dict[str, torch.Tensor], lists: Dict[str, np.ndarray], dims: Dict[str, int]):
    """The float64 forward with fixed selections.  x: q, k [B,H,T,d_qk], v
    [B,H,T,d_v], alpha, beta [B,H,T], C1, C2 [H,n,d_h], M0 [B,H,N,d_v] (float64
    tensors, possibly requiring grad); lists: idx_w [B,H,T,W], idx_r [B,H,T,R]
    (the oracle's selections).  Returns o [B,H,T,d_v] and M_T [B,H,N,d_v]."""
    B, H, T = dims['B'], dims['H'], dims['T']
    n, dh = dims['n_sub'], dims['d_qk'] // 2
    os_, Ms = [], []
    for b in range(B):
        ob, Mb = [], []
        for h in range(H):
            # only the rows the head ever selects take part: a compact table of
            # them (gathered from M0, so its gradient flows back to M0)
            iw = lists['idx_w'][b, h].astype(np.int64)
            ir = lists['idx_r'][b, h].astype(np.int64)
            rows = np.unique(np.concatenate([iw.reshape(-1), ir.reshape(-1)]))
            rows_t = torch.as_tensor(rows)
            M = x['M0'][b, h][rows_t]
            C1, C2 = x['C1'][h], x['C2'][h]
            oh = []
            for t in range(T):
                kt, qt = x['k'][b, h, t], x['q'][b, h, t]
                ws = torch.as_tensor(iw[t])
                rs = torch.as_tensor(ir[t])
                cw = torch.as_tensor(np.searchsorted(rows, iw[t]))
                cr = torch.as_tensor(np.searchsorted(rows, ir[t]))
                sw = (C1[ws // n] @ kt[:dh]) + (C2[ws % n] @ kt[dh:])
                sr = (C1[rs // n] @ qt[:dh]) + (C2[rs % n] @ qt[dh:])
                w = torch.softmax(sw, 0)
                u = torch.softmax(sr, 0)
                c = x['beta'][b, h, t] * w
                Mt = x['alpha'][b, h, t] * M[cw]
                new = (1.0 - c)[:, None] * Mt + c[:, None] * x['v'][b, h, t][None, :]
                M = M.index_copy(0, cw, new)
                oh.append(u @ M[cr])
            ob.append(torch.stack(oh) if oh else torch.zeros(0, x['v'].shape[-1],
                                                             dtype=torch.float64))
            Mb.append(x['M0'][b, h].index_copy(0, rows_t, M))
        os_.append(torch.stack(ob))
        Ms.append(torch.stack(Mb))
    return torch.stack(os_), torch.stack(Ms)


NAMES = ('q', 'k', 'v', 'alpha', 'beta', 'C1', 'C2', 'M0')


def grads(inp: Dict[str, np.ndarray], lists: Dict[str, np.ndarray], dims: Dict[str, int],
          do: np.ndarray, dM: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Gradients of L = sum(o * do) + sum(M_T * dM) with respect to q, k, v,
    alpha, beta, C1, C2 and M0 (float64 numpy arrays), at the given selections."""
    x = {nm: _t64(inp[nm], True) for nm in NAMES}
    o, MT = forward64(x, lists, dims)
    L = (o * _t64(do)).sum()
    if dM is not None:
        L = L + (MT * _t64(dM)).sum()
    g = torch.autograd.grad(L, [x[nm] for nm in NAMES], allow_unused=True)
    return {nm: (gi.numpy() if gi is not None else np.zeros_like(inp[nm], dtype=np.float64))
            for nm, gi in zip(NAMES, g)}


def loss64(inp: Dict[str, np.ndarray], lists, dims, do, dM=None) -> float:
    """L of grads(), for finite differences."""
    with torch.no_grad():
        o, MT = forward64({nm: _t64(inp[nm]) for nm in NAMES}, lists, dims)
        L = (o * _t64(do)).sum()
        if dM is not None:
            L = L + (MT * _t64(dM)).sum()
    return float(L)
