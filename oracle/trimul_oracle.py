"""fp64 numpy oracle of the full triangle multiplicative update (test
infrastructure only: the tests, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py`` may use it; it shares no code with the CUDA library).

The pages name triangle multiplication beside triangle attention as the second
pair-stack operation their kernels accelerate ("TurboPairFormer accelera fino a
1,73x l'addestramento di OpenFold3 nei test", sections "Dove si impiega il
tempo" and "Benchmark di addestramento") but print no formula. The reading
taken is the standard AlphaFold-family update, per pair position p = (i, j) of
the pair representation z [N][N][cz]:

  x      = LayerNorm(z)                              over cz (biased variance)
  [ap | ag | bp | bg | gl] = x W_in + b_in           W_in [cz][4c + cz]
  a      = sigmoid(ag) * ap,   b = sigmoid(bg) * bp   [N][N][c]
  t[i,j] = sum_k a[i,k] * b[j,k]                     outgoing edges
  t[i,j] = sum_k a[k,i] * b[k,j]                     incoming edges
  u      = LayerNorm_out(t)                          over c
  y      = sigmoid(gl) * (u W_o + b_o)               W_o [c][cz]

The backward is the gradient of L = sum(dy * y), written out by hand from the
chain rule in the reverse order of the steps. Inputs are the values the GPU
receives (bf16 or fp32, widened without change); every computation is fp64.
"""

from __future__ import annotations

import numpy as np

from .proj_oracle import layer_norm, layer_norm_bwd

OUTGOING, INCOMING = 0, 1


def _f64(a):
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.asarray(a, dtype=np.float64)


def _sigmoid(v):
    return 1.0 / (1.0 + np.exp(-v))


def contract(a, b, direction):
    """t [N][N][c] from a, b [N][N][c] (the sums written out above)."""
    if direction == OUTGOING:
        return np.einsum("ikc,jkc->ijc", a, b)
    return np.einsum("kic,kjc->ijc", a, b)


def update_fwd(z, p, direction, eps=1e-5):
    """z [N][N][cz]; p: dict of ln_gamma, ln_beta [cz], w_in [cz][4c+cz], b_in,
    ln_out_gamma, ln_out_beta [c], w_o [c][cz], b_o [cz]. Returns y and a dict of
    the intermediate values the backward uses."""
    z = _f64(z)
    N, _, cz = z.shape
    w_in = _f64(p["w_in"])
    c = (w_in.shape[1] - cz) // 4
    x, _, _ = layer_norm(z.reshape(N * N, cz), p["ln_gamma"], p["ln_beta"], eps)
    pre = x @ w_in + _f64(p["b_in"])
    ap, ag, bp, bg, gl = (pre[:, 0:c], pre[:, c:2 * c], pre[:, 2 * c:3 * c],
                          pre[:, 3 * c:4 * c], pre[:, 4 * c:])
    a = _sigmoid(ag) * ap
    b = _sigmoid(bg) * bp
    t = contract(a.reshape(N, N, c), b.reshape(N, N, c), direction).reshape(N * N, c)
    u, _, _ = layer_norm(t, p["ln_out_gamma"], p["ln_out_beta"], eps)
    h = u @ _f64(p["w_o"]) + _f64(p["b_o"])
    g = _sigmoid(gl)
    y = g * h
    cache = dict(x=x, pre=pre, a=a, b=b, t=t, u=u, h=h, g=g, N=N, c=c, cz=cz)
    return y.reshape(N, N, cz), cache


def update_bwd(z, p, direction, dy, eps=1e-5):
    """Gradients of L = sum(dy * y): dict(dz, and d<name> for every parameter)."""
    _, k = update_fwd(z, p, direction, eps)
    N, c, cz = k["N"], k["c"], k["cz"]
    dy = _f64(dy).reshape(N * N, cz)
    w_in, w_o = _f64(p["w_in"]), _f64(p["w_o"])
    # y = g * h, g = sigmoid(gl), h = u W_o + b_o
    dh = dy * k["g"]
    dgl = dy * k["h"] * k["g"] * (1.0 - k["g"])
    d_w_o = k["u"].T @ dh
    d_b_o = dh.sum(axis=0)
    du = dh @ w_o.T
    dt, d_ln_out_gamma, d_ln_out_beta = layer_norm_bwd(k["t"], p["ln_out_gamma"], eps, du)
    # t = contract(a, b): t is bilinear in a and b
    a3, b3, dt3 = k["a"].reshape(N, N, c), k["b"].reshape(N, N, c), dt.reshape(N, N, c)
    if direction == OUTGOING:
        da = np.einsum("ijc,jkc->ikc", dt3, b3)
        db = np.einsum("ijc,ikc->jkc", dt3, a3)
    else:
        da = np.einsum("ijc,kjc->kic", dt3, b3)
        db = np.einsum("ijc,kic->kjc", dt3, a3)
    da, db = da.reshape(N * N, c), db.reshape(N * N, c)
    pre = k["pre"]
    ap, ag, bp, bg = pre[:, 0:c], pre[:, c:2 * c], pre[:, 2 * c:3 * c], pre[:, 3 * c:4 * c]
    sa, sb = _sigmoid(ag), _sigmoid(bg)
    dpre = np.concatenate([da * sa, da * ap * sa * (1.0 - sa),
                           db * sb, db * bp * sb * (1.0 - sb), dgl], axis=1)
    d_w_in = k["x"].T @ dpre
    d_b_in = dpre.sum(axis=0)
    dx = dpre @ w_in.T
    dz, d_ln_gamma, d_ln_beta = layer_norm_bwd(_f64(z).reshape(N * N, cz), p["ln_gamma"], eps,
                                               dx)
    return dict(dz=dz.reshape(N, N, cz), ln_gamma=d_ln_gamma, ln_beta=d_ln_beta, w_in=d_w_in,
                b_in=d_b_in, ln_out_gamma=d_ln_out_gamma, ln_out_beta=d_ln_out_beta, w_o=d_w_o,
                b_o=d_b_o)
