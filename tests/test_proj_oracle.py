"""Pins of the projection oracle (CPU, fp64). The pages print neither the
LayerNorm nor the projections, so the oracle is pinned to what fixes them
independently of how it is coded: torch's own fp64 layer_norm and autograd
(a library routine, not a retyping of the oracle's formulas), central finite
differences, and invariants of LayerNorm (zero mean and unit variance of the
normalised rows, invariance to a per-row shift and, with eps = 0, to a
per-row scale, hence gradients orthogonal to those directions). A mutation
test plants plausible mistakes in the oracle's source and checks that each one
trips a pin."""

import importlib.util
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import proj_oracle

ROWS, CZ, H, C = 13, 16, 3, 4          # small, non-square everywhere
HC = H * C
EPS = 1e-5


def rand(shape, seed, scale=1.0, shift=0.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale + shift


def case():
    return dict(z=rand((ROWS, CZ), 1, 2.0, 0.5), gamma=rand(CZ, 2, 0.5, 1.0),
                beta=rand(CZ, 3, 0.3), w_qkvg=rand((CZ, 4 * HC), 4, 0.3),
                b_g=rand(HC, 5, 0.2), w_b=rand((CZ, H), 6, 0.3), w_o=rand((HC, CZ), 7, 0.3),
                b_o=rand(CZ, 8, 0.2), o=rand((ROWS, HC), 9),
                d=[rand((ROWS, HC), 10 + i) for i in range(4)], dbias=rand((H, ROWS), 14),
                dy=rand((ROWS, CZ), 15))


def torch_reference(p):
    """The same block through torch.nn.functional.layer_norm and autograd, fp64."""
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True)
         for k, v in p.items() if k not in ("d",)}
    x = torch.nn.functional.layer_norm(t["z"], (CZ,), t["gamma"], t["beta"], EPS)
    proj = x @ t["w_qkvg"]
    q, k, v, g = proj[:, :HC], proj[:, HC:2 * HC], proj[:, 2 * HC:3 * HC], proj[:, 3 * HC:]
    g = g + t["b_g"]
    bias = (x @ t["w_b"]).T
    y = t["o"] @ t["w_o"] + t["b_o"]
    d = [torch.tensor(a) for a in p["d"]]
    L = ((d[0] * q).sum() + (d[1] * k).sum() + (d[2] * v).sum() + (d[3] * g).sum() +
         (t["dbias"] * bias).sum() + (t["dy"] * y).sum())
    L.backward()
    grad = {k: t[k].grad.numpy() for k in ("z", "gamma", "beta", "w_qkvg", "b_g", "w_b",
                                             "o", "w_o", "b_o")}
    return {"x": x.detach().numpy(), "q": q.detach().numpy(), "k": k.detach().numpy(),
            "v": v.detach().numpy(), "gate": g.detach().numpy(), "bias": bias.detach().numpy(),
            "y": y.detach().numpy()}, grad


def run(mod, p):
    f = mod.proj_in_fwd(p["z"], p["gamma"], p["beta"], p["w_qkvg"], p["b_g"], p["w_b"], EPS)
    b = mod.proj_in_bwd(p["z"], p["gamma"], p["beta"], p["w_qkvg"], p["w_b"], EPS, *p["d"],
                        p["dbias"])
    y = mod.proj_out_fwd(p["o"], p["w_o"], p["b_o"])
    ob = mod.proj_out_bwd(p["o"], p["w_o"], p["dy"])
    return f, b, y, ob


def pins(mod=proj_oracle):
    """Every pin; returns the names of those that fail (empty = all hold)."""
    failed = []
    p = case()
    try:
        f, b, y, ob = run(mod, p)
    except Exception as e:                           # a mistake that breaks shapes
        return [f"raises {type(e).__name__}"]
    ref, grad = torch_reference(p)

    def close(a, r, name, tol=1e-10):
        if np.shape(a) != np.shape(r) or not np.allclose(a, r, rtol=tol, atol=tol):
            failed.append(name)

    # torch's fp64 layer_norm and autograd
    for k in ("x", "q", "k", "v", "gate", "bias"):
        close(f[k], ref[k], f"torch-{k}")
    close(y, ref["y"], "torch-y")
    close(b["dz"], grad["z"], "torch-dz")
    for k in ("dgamma", "dbeta", "dw_qkvg", "db_g", "dw_b"):
        close(b[k], grad[k[1:]], f"torch-{k}")
    for k in ("do", "dw_o", "db_o"):
        close(ob[k], grad[k[1:]], f"torch-{k}")

    # LayerNorm invariants: normalised rows (gamma = 1, beta = 0) have zero mean
    # and variance var / (var + eps); a per-row shift changes nothing, nor (eps = 0)
    # a per-row positive scale
    one, zero = np.ones(CZ), np.zeros(CZ)
    xh, mean, rstd = mod.layer_norm(p["z"], one, zero, EPS)
    var = p["z"].var(axis=1)
    if not (np.allclose(xh.mean(axis=1), 0, atol=1e-12) and
            np.allclose(xh.var(axis=1), var / (var + EPS), rtol=1e-12)):
        failed.append("ln-moments")
    if not np.allclose(mean, p["z"].mean(axis=1), rtol=1e-12):
        failed.append("ln-mean")
    shift = rand((ROWS, 1), 20, 3.0)
    if not np.allclose(mod.layer_norm(p["z"] + shift, p["gamma"], p["beta"], EPS)[0], f["x"],
                       rtol=1e-10, atol=1e-10):
        failed.append("ln-shift")
    scale = np.exp(rand((ROWS, 1), 21))
    if not np.allclose(mod.layer_norm(p["z"] * scale, p["gamma"], p["beta"], 0.0)[0],
                       mod.layer_norm(p["z"], p["gamma"], p["beta"], 0.0)[0], rtol=1e-10,
                       atol=1e-10):
        failed.append("ln-scale")
    # so dz is orthogonal to the constant row, and (eps = 0) to the centred row
    if not np.allclose(b["dz"].sum(axis=1), 0, atol=1e-10):
        failed.append("dz-shift")
    b0 = mod.proj_in_bwd(p["z"], p["gamma"], p["beta"], p["w_qkvg"], p["w_b"], 0.0, *p["d"],
                         p["dbias"])
    zc = p["z"] - p["z"].mean(axis=1, keepdims=True)
    if not np.allclose((b0["dz"] * zc).sum(axis=1), 0, atol=1e-9):
        failed.append("dz-scale")

    # central finite differences of L on a few coordinates of every input
    def loss(q):
        ff = mod.proj_in_fwd(q["z"], q["gamma"], q["beta"], q["w_qkvg"], q["b_g"], q["w_b"], EPS)
        yy = mod.proj_out_fwd(q["o"], q["w_o"], q["b_o"])
        return (sum(np.sum(d * ff[k]) for d, k in zip(q["d"], ("q", "k", "v", "gate"))) +
                np.sum(q["dbias"] * ff["bias"]) + np.sum(q["dy"] * yy))

    analytic = {"z": b["dz"], "gamma": b["dgamma"], "beta": b["dbeta"], "w_qkvg": b["dw_qkvg"],
                "b_g": b["db_g"], "w_b": b["dw_b"], "o": ob["do"], "w_o": ob["dw_o"],
                "b_o": ob["db_o"]}
    rng = np.random.default_rng(30)
    h = 1e-5
    for name, g in analytic.items():
        for _ in range(3):
            idx = tuple(int(rng.integers(0, s)) for s in p[name].shape)
            qp = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in p.items()}
            qm = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in p.items()}
            qp[name][idx] += h
            qm[name][idx] -= h
            fd = (loss(qp) - loss(qm)) / (2 * h)
            if np.shape(g) != p[name].shape or not np.isclose(fd, g[idx], rtol=1e-6, atol=1e-7):
                failed.append(f"fd-{name}")
                break
    return failed


def test_oracle_meets_every_pin():
    assert pins() == []


def test_package_exports_the_oracle():
    assert oracle.proj_in_fwd is proj_oracle.proj_in_fwd
    assert oracle.proj_out_bwd is proj_oracle.proj_out_bwd


MUTANTS = {
    "unbiased variance": ("var = ((z - mean[..., None]) ** 2).mean(axis=-1)",
                          "var = ((z - mean[..., None]) ** 2).sum(axis=-1) / (z.shape[-1] - 1)"),
    "eps outside the root": ("rstd = 1.0 / np.sqrt(var + eps)",
                             "rstd = 1.0 / (np.sqrt(var) + eps)"),
    "k and v swapped": ('"k": proj[:, hc:2 * hc], "v": proj[:, 2 * hc:3 * hc]',
                        '"k": proj[:, 2 * hc:3 * hc], "v": proj[:, hc:2 * hc]'),
    "gate bias dropped": ('"gate": proj[:, 3 * hc:4 * hc] + _f64(b_g)',
                          '"gate": proj[:, 3 * hc:4 * hc]'),
    "dz without the mean term": ("u - u.mean(axis=-1, keepdims=True) - xhat",
                                 "u - xhat"),
    "dz without the variance term": (
        "dz = rstd * (u - u.mean(axis=-1, keepdims=True) - xhat * (u * xhat).mean(axis=-1, keepdims=True))",
        "dz = rstd * (u - u.mean(axis=-1, keepdims=True))"),
    "dgamma from x": ("(dx * xhat).sum(axis=0)", "(dx * (xhat * _f64(gamma))).sum(axis=0)"),
    "bias path missing from dx": ("dx = dp @ _f64(w_qkvg).T + dbias.T @ _f64(w_b).T",
                                  "dx = dp @ _f64(w_qkvg).T"),
    "weight gradient from z": ('"dw_qkvg": x.T @ dp', '"dw_qkvg": _f64(z).T @ dp'),
    "bias weight gradient transposed": ('"dw_b": x.T @ dbias.T', '"dw_b": (dbias @ x).T[:, ::-1]'),
    "output bias gradient averaged": ('"db_o": dy.sum(axis=0)', '"db_o": dy.mean(axis=0)'),
    "output weight gradient from dy alone": ('"dw_o": _f64(o).T @ dy',
                                             '"dw_o": _f64(o).T @ np.sign(dy)'),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_mutant_fails_a_pin(name, tmp_path):
    src = open(proj_oracle.__file__).read()
    old, new = MUTANTS[name]
    assert old in src, name
    path = tmp_path / "mutant_proj_oracle.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("mutant_proj_oracle", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    assert pins(mod) != [], f"mutant '{name}' passes every pin"
