"""fp64 numpy oracle of the steps either side of triangle attention (test
infrastructure only: the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may use it; it shares no code with the CUDA library).

The pages name these steps without printing them: LayerNorm takes 14% of
AlphaFold training time at 10% of its theoretical speed before optimisation
("알파폴드 초기 학습 시간을 10시간으로 단축하는 ScaleFold", Stats), and the
gated self-attention is fused with the projections around it ("HelixFold: An
Efficient Implementation of AlphaFold2 using PaddlePaddle", proposed methods:
fused gated self-attention). The reading taken here is the standard
AlphaFold-family triangle attention block, per pair position (a row of the pair
representation z, cz channels):

  input side   x = LayerNorm(z) = (z - mean(z)) / sqrt(var(z) + eps) * gamma + beta
               (mean and the biased variance over the cz channels)
               q = x Wq, k = x Wk, v = x Wv          no bias, H heads of c channels
               g = x Wg + bg                         gate logits (the sigmoid is the
                                                     attention's)
               b[h] = x wb[:, h]                     pair bias, no bias term
  output side  y = o Wo + bo                         o: the gated attention output

Wq|Wk|Wv|Wg are the four column blocks of one [cz][4*H*c] matrix. Every
backward is the gradient of L = sum(dq q) + sum(dk k) + sum(dv v) + sum(dg g)
+ sum(db b) (input side) or L = sum(dy y) (output side), written out by hand
from the chain rule. Inputs are the values the GPU receives (bf16 or fp32,
widened without change); every computation and result is fp64.
"""

from __future__ import annotations

import numpy as np


def _f64(a):
    if hasattr(a, "detach"):                  # a torch tensor (bf16 included)
        a = a.detach().cpu().double().numpy()
    return np.asarray(a, dtype=np.float64)


def layer_norm(z, gamma, beta, eps):
    """x, mean, rstd of LayerNorm over the last axis (biased variance)."""
    z = _f64(z)
    mean = z.mean(axis=-1)
    var = ((z - mean[..., None]) ** 2).mean(axis=-1)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = (z - mean[..., None]) * rstd[..., None]
    return xhat * _f64(gamma) + _f64(beta), mean, rstd


def proj_in_fwd(z, gamma, beta, w_qkvg, b_g, w_b, eps):
    """z [rows][cz] -> dict(x, mean, rstd, q, k, v, gate [rows][H*c], bias [H][rows]).

    w_qkvg [cz][4*H*c] holds Wq, Wk, Wv, Wg side by side; b_g [H*c]; w_b [cz][H]."""
    x, mean, rstd = layer_norm(z, gamma, beta, eps)
    hc = _f64(w_qkvg).shape[1] // 4
    proj = x @ _f64(w_qkvg)
    out = {"x": x, "mean": mean, "rstd": rstd,
           "q": proj[:, 0:hc], "k": proj[:, hc:2 * hc], "v": proj[:, 2 * hc:3 * hc],
           "gate": proj[:, 3 * hc:4 * hc] + _f64(b_g),
           "bias": (x @ _f64(w_b)).T}
    return out


def layer_norm_bwd(z, gamma, eps, dx):
    """dz, dgamma, dbeta of x = LayerNorm(z) * gamma + beta given dL/dx.

    With xhat = (z - mean) * rstd and u = dx * gamma, the chain rule through the
    mean and the variance gives dz = rstd * (u - mean(u) - xhat * mean(u * xhat))."""
    z, dx = _f64(z), _f64(dx)
    mean = z.mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(((z - mean) ** 2).mean(axis=-1, keepdims=True) + eps)
    xhat = (z - mean) * rstd
    u = dx * _f64(gamma)
    dz = rstd * (u - u.mean(axis=-1, keepdims=True) - xhat * (u * xhat).mean(axis=-1, keepdims=True))
    return dz, (dx * xhat).sum(axis=0), dx.sum(axis=0)


def proj_in_bwd(z, gamma, beta, w_qkvg, w_b, eps, dq, dk, dv, dgate, dbias):
    """Gradients of the input side: dict(dz, dgamma, dbeta, dw_qkvg, db_g, dw_b)."""
    x, _, _ = layer_norm(z, gamma, beta, eps)
    dp = np.concatenate([_f64(dq), _f64(dk), _f64(dv), _f64(dgate)], axis=1)
    dbias = _f64(dbias)                                   # [H][rows]
    dx = dp @ _f64(w_qkvg).T + dbias.T @ _f64(w_b).T
    dz, dgamma, dbeta = layer_norm_bwd(z, gamma, eps, dx)
    return {"dz": dz, "dgamma": dgamma, "dbeta": dbeta,
            "dw_qkvg": x.T @ dp, "db_g": _f64(dgate).sum(axis=0), "dw_b": x.T @ dbias.T}


def proj_out_fwd(o, w_o, b_o):
    """y [rows][cz] = o [rows][H*c] Wo [H*c][cz] + bo [cz]."""
    return _f64(o) @ _f64(w_o) + _f64(b_o)


def proj_out_bwd(o, w_o, dy):
    """Gradients of the output side: dict(do, dw_o, db_o)."""
    dy = _f64(dy)
    return {"do": dy @ _f64(w_o).T, "dw_o": _f64(o).T @ dy, "db_o": dy.sum(axis=0)}
