"""Pins for the fp64 oracle (CPU only).

The oracle is checked against things other than itself:
  * a composition of library routines: torch's fp64 scaled_dot_product_attention
    and sigmoid, differentiated by autograd (forward and all five gradients);
  * central finite differences (Richardson-extrapolated) of the oracle's own
    forward, which pin every analytic gradient;
  * an independent numpy backward through the explicit softmax Jacobian
    (diag(p) - p p^T), not through the row-sum shortcut the oracle uses;
  * closed forms, invariants and symmetries that hold for any correct
    implementation (probability rows sum to one, key-permutation invariance,
    bias-shift invariance, one-key and N=1 cases, zero row sums of dbias);
  * the ending-node variant against the starting node on transposed inputs.

Every check is a function of an optional oracle library handle, so
``test_mutants_are_caught`` can build deliberately broken copies of the oracle
(a dropped term, a flipped sign, a wrong index, a transposed operand) and show
that each one fails at least one pin.
"""

import os
import re
import shutil
import tempfile

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from tri_inputs import ENDING, STARTING, full_mask, make_inputs

TOL = 1e-12


def tiny(N=5, H=2, C=4, seed=0, bias_std=1.0, mask="none"):
    """bf16-representable values widened to float32, so that x +- 2^-8 and
    x +- 2^-9 stay exact for the finite-difference pins."""
    d = make_inputs(N, H, C, dtype="bf16", seed=seed, bias_std=bias_std, mask=mask)
    out = {}
    for key, val in d.items():
        if torch.is_tensor(val) and val.is_floating_point():
            out[key] = val.to(torch.float32)
        else:
            out[key] = val
    return out


def args(d):
    return d["q"], d["k"], d["v"], d["bias"], d["gate"]


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = max(np.linalg.norm(b.ravel()), 1e-300)
    return np.linalg.norm((a - b).ravel()) / den


def close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(1.0, np.max(np.abs(b)) if b.size else 0.0)
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} (scale {scale:.3e})"


def to_variant_frame(t, variant):
    """Pair tensor [a, b, H, C] in storage layout -> [row, query, H, C]."""
    return t if variant == STARTING else t.transpose(0, 1)


# ----------------------------------------------------------------------------
# library composition: torch SDPA (fp64) * sigmoid, autograd for the gradients
# ----------------------------------------------------------------------------

def torch_reference(d, mask, variant):
    """out, lse and the five gradients from torch library routines, fp64, with
    the same conventions as the oracle (pair outputs in the variant frame,
    dbias in storage layout)."""
    leaves = {n: d[n].to(torch.float64).clone().requires_grad_(True)
              for n in ("q", "k", "v", "gate", "bias")}
    q, k, v, g = (to_variant_frame(leaves[n], variant) for n in ("q", "k", "v", "gate"))
    b = leaves["bias"] if variant == STARTING else leaves["bias"].transpose(1, 2)
    dout = to_variant_frame(d["dout"].to(torch.float64), variant)
    N, _, H, C = q.shape
    mu = torch.zeros((N, 1, 1, N), dtype=torch.float64)
    if mask is not None:
        m = mask.to(torch.bool)
        if m.dim() == 1:
            m = m.expand(N, N)
        mu = torch.where(m, 0.0, float("-inf")).to(torch.float64).reshape(N, 1, 1, N)
    attn = b.unsqueeze(0) + mu                                   # [r, h, x, y]
    Q, K, V = (t.permute(0, 2, 1, 3) for t in (q, k, v))         # [r, h, x, c]
    O = F.scaled_dot_product_attention(Q, K, V, attn_mask=attn)  # scale 1/sqrt(C)
    out = torch.sigmoid(g) * O.permute(0, 2, 1, 3)
    loss = (dout * out).sum()
    loss.backward()
    lse = torch.logsumexp(torch.einsum("rhxc,rhyc->rhxy", Q, K) / np.sqrt(C) + attn, dim=-1)
    grads = {n: to_variant_frame(leaves[n].grad, variant).detach().numpy()
             for n in ("q", "k", "v", "gate")}
    return (out.detach().numpy(), lse.detach().numpy(), grads["q"], grads["k"], grads["v"],
            grads["gate"], leaves["bias"].grad.detach().numpy())


def check_library_composition(lib=None, variant=STARTING, mask_kind="random:2", N=6):
    d = tiny(N=N, H=2, C=4, seed=3, bias_std=np.sqrt(2.0), mask=mask_kind)
    ref = torch_reference(d, d["mask"], variant)
    out, lse = oracle.fwd(*args(d), d["mask"], variant, lib=lib)
    dq, dk, dv, dg, db = oracle.bwd(*args(d), d["dout"], d["mask"], variant, lib=lib)
    for name, a, b in zip(("out", "lse", "dq", "dk", "dv", "dgate", "dbias"),
                          (out, lse, dq, dk, dv, dg, db), ref):
        close(a, b, 1e-11, name)


# ----------------------------------------------------------------------------
# finite differences of the oracle's forward
# ----------------------------------------------------------------------------

def check_finite_differences(lib=None, variant=STARTING, N=4, H=2, C=4):
    d = tiny(N=N, H=H, C=C, seed=11, mask="random:1")
    mask = d["mask"]
    dout = d["dout"].to(torch.float64).numpy()

    def loss(dd):
        out, _ = oracle.fwd(*args(dd), mask, variant, lib=lib)
        out_st = oracle.to_storage(out, variant)
        return float(np.sum(dout * out_st))

    dq, dk, dv, dg, db = oracle.bwd(*args(d), d["dout"], mask, variant, lib=lib)
    analytic = {"q": oracle.to_storage(dq, variant), "k": oracle.to_storage(dk, variant),
                "v": oracle.to_storage(dv, variant), "gate": oracle.to_storage(dg, variant),
                "bias": db}
    h = 2.0 ** -8
    for name in ("q", "k", "v", "gate", "bias"):
        base = d[name]
        flat = base.reshape(-1)
        fd = np.zeros(flat.numel())
        for e in range(flat.numel()):
            vals = []
            for step in (h, -h, h / 2, -h / 2):
                pert = flat.clone()
                pert[e] = pert[e] + step
                assert float(pert[e]) - float(flat[e]) == step, "perturbation not exact"
                dd = dict(d)
                dd[name] = pert.reshape(base.shape)
                vals.append(loss(dd))
            d1 = (vals[0] - vals[1]) / (2 * h)
            d2 = (vals[2] - vals[3]) / h
            fd[e] = (4 * d2 - d1) / 3
        close(analytic[name].reshape(-1), fd, 1e-7, f"d{name} vs finite differences")


# ----------------------------------------------------------------------------
# explicit-Jacobian backward in numpy
# ----------------------------------------------------------------------------

def jacobian_reference(d, variant):
    q, k, v, g, do = (to_variant_frame(d[n], variant).to(torch.float64).numpy()
                      for n in ("q", "k", "v", "gate", "dout"))
    b = d["bias"].to(torch.float64).numpy()
    if variant == ENDING:
        b = b.transpose(0, 2, 1)
    N, _, H, C = q.shape
    mask = d["mask"]
    keep = np.ones((N, N), dtype=bool)
    if mask is not None:
        m = mask.numpy().astype(bool)
        keep = np.broadcast_to(m, (N, N)) if m.ndim == 1 else m
    out = np.zeros_like(q); dq = np.zeros_like(q); dk = np.zeros_like(q)
    dv = np.zeros_like(q); dg = np.zeros_like(q); db = np.zeros_like(b)
    sig = 1.0 / (1.0 + np.exp(-g))
    for r in range(N):
        for h in range(H):
            S = q[r, :, h, :] @ k[r, :, h, :].T / np.sqrt(C) + b[h]
            S = np.where(keep[r][None, :], S, -np.inf)
            P = np.exp(S - S.max(axis=1, keepdims=True))
            P = P / P.sum(axis=1, keepdims=True)
            U = P @ v[r, :, h, :]
            out[r, :, h, :] = sig[r, :, h, :] * U
            dU = do[r, :, h, :] * sig[r, :, h, :]
            dg[r, :, h, :] = do[r, :, h, :] * U * sig[r, :, h, :] * (1 - sig[r, :, h, :])
            dP = dU @ v[r, :, h, :].T
            dS = np.zeros_like(P)
            for x in range(N):
                J = np.diag(P[x]) - np.outer(P[x], P[x])
                dS[x] = J @ dP[x]
            dq[r, :, h, :] = dS @ k[r, :, h, :] / np.sqrt(C)
            dk[r, :, h, :] = dS.T @ q[r, :, h, :] / np.sqrt(C)
            dv[r, :, h, :] = P.T @ dU
            db[h] += dS
    if variant == ENDING:
        db = db.transpose(0, 2, 1)
    return out, dq, dk, dv, dg, db


def check_jacobian(lib=None, variant=STARTING):
    d = tiny(N=7, H=2, C=8, seed=5, bias_std=np.sqrt(2.0), mask="random:2")
    ref = jacobian_reference(d, variant)
    out, _ = oracle.fwd(*args(d), d["mask"], variant, lib=lib)
    got = (out,) + oracle.bwd(*args(d), d["dout"], d["mask"], variant, lib=lib)
    for name, a, b in zip(("out", "dq", "dk", "dv", "dgate", "dbias"), got, ref):
        close(a, b, TOL, name)


# ----------------------------------------------------------------------------
# probabilities, closed forms, invariants, symmetries
# ----------------------------------------------------------------------------

def check_probabilities(lib=None):
    d = tiny(N=8, H=2, C=4, seed=2, mask="random:3")
    keep = d["mask"].numpy().astype(bool)
    for variant in (STARTING, ENDING):
        for r in (0, 5):
            for h in range(2):
                P = oracle.probs(d["q"], d["k"], d["v"], d["bias"], d["mask"], variant, r, h,
                                 lib=lib)
                close(P.sum(axis=1), np.ones(8), 1e-13, "row sums")
                assert np.all(P[:, ~keep] == 0.0), "masked keys must get zero probability"
                assert np.all(P[:, keep] > 0.0)
    # lse is the log of the softmax normaliser: p = exp(s - lse) must sum to one
    out, lse = oracle.fwd(*args(d), d["mask"], STARTING, lib=lib)
    q, k, b = (d[n].to(torch.float64).numpy() for n in ("q", "k", "bias"))
    for r in (1, 6):
        for h in range(2):
            s = q[r, :, h, :] @ k[r, :, h, :].T / 2.0 + b[h]
            z = np.exp(s[:, keep] - lse[r, h][:, None]).sum(axis=1)
            close(z, np.ones(8), 1e-13, "exp(s - lse) row sums")


def check_closed_forms(lib=None):
    N, H, C = 6, 2, 4
    d = tiny(N=N, H=H, C=C, seed=9)
    sig = torch.sigmoid(d["gate"].to(torch.float64)).numpy()
    v = d["v"].to(torch.float64).numpy()
    # (i) q = 0 and b = 0: uniform attention, out = sigmoid(g) * mean_y v, lse = log N
    dz = dict(d)
    dz["q"] = torch.zeros_like(d["q"])
    dz["bias"] = torch.zeros_like(d["bias"])
    out, lse = oracle.fwd(*args(dz), None, STARTING, lib=lib)
    close(out, sig * v.mean(axis=1, keepdims=True), TOL, "uniform attention")
    close(lse, np.full((N, H, N), np.log(N)), TOL, "uniform lse")
    # (ii) a single key kept: p is one-hot
    ystar = 4
    m = torch.zeros(N, dtype=torch.uint8)
    m[ystar] = 1
    out, lse = oracle.fwd(*args(d), m, STARTING, lib=lib)
    close(out, sig * v[:, ystar:ystar + 1], TOL, "one key kept: out")
    dq, dk, dv, dg, db = oracle.bwd(*args(d), d["dout"], m, STARTING, lib=lib)
    close(dq, np.zeros_like(dq), TOL, "one key kept: dq")
    close(dk, np.zeros_like(dk), TOL, "one key kept: dk")
    close(db, np.zeros_like(db), TOL, "one key kept: dbias")
    du = d["dout"].to(torch.float64).numpy() * sig
    exp_dv = np.zeros_like(dv)
    exp_dv[:, ystar] = du.sum(axis=1)
    close(dv, exp_dv, TOL, "one key kept: dv")
    # (iii) N = 1
    d1 = tiny(N=1, H=H, C=C, seed=4)
    out, lse = oracle.fwd(*args(d1), None, STARTING, lib=lib)
    close(out, torch.sigmoid(d1["gate"].double()).numpy() * d1["v"].double().numpy(), TOL,
          "N=1 out")
    dq, dk, dv, dg, db = oracle.bwd(*args(d1), d1["dout"], None, STARTING, lib=lib)
    for name, a in (("dq", dq), ("dk", dk), ("dbias", db)):
        close(a, np.zeros_like(a), TOL, f"N=1 {name}")
    # (iv) shifting a bias row by a constant changes only lse
    shift = torch.tensor([0.5, -1.25, 2.0, 0.0, 0.75, -0.5], dtype=torch.float32)
    ds = dict(d)
    ds["bias"] = d["bias"] + shift.reshape(1, N, 1)
    out0, lse0 = oracle.fwd(*args(d), None, STARTING, lib=lib)
    out1, lse1 = oracle.fwd(*args(ds), None, STARTING, lib=lib)
    close(out1, out0, 1e-13, "bias shift: out")
    close(lse1 - lse0, np.broadcast_to(shift.double().numpy(), lse0.shape), 1e-13,
          "bias shift: lse")
    g0 = oracle.bwd(*args(d), d["dout"], None, STARTING, lib=lib)
    g1 = oracle.bwd(*args(ds), d["dout"], None, STARTING, lib=lib)
    for name, a, b in zip(("dq", "dk", "dv", "dgate", "dbias"), g1, g0):
        close(a, b, 1e-12, f"bias shift: {name}")


def check_invariants(lib=None):
    N, H, C = 7, 2, 4
    d = tiny(N=N, H=H, C=C, seed=21, bias_std=np.sqrt(2.0), mask="random:2")
    dq, dk, dv, dg, db = oracle.bwd(*args(d), d["dout"], d["mask"], STARTING, lib=lib)
    close(db.sum(axis=2), np.zeros((H, N)), TOL, "sum_y dbias")
    sig = torch.sigmoid(d["gate"].double()).numpy()
    du = d["dout"].double().numpy() * sig
    close(dv.sum(axis=1), du.sum(axis=1), TOL, "sum_y dv = sum_x du")
    # out is linear in v
    d2 = dict(d)
    d2["v"] = d["v"] * 2.0
    o1, _ = oracle.fwd(*args(d), d["mask"], STARTING, lib=lib)
    o2, _ = oracle.fwd(*args(d2), d["mask"], STARTING, lib=lib)
    close(o2, 2.0 * o1, TOL, "out linear in v")


def check_permutation(lib=None):
    N, H, C = 7, 2, 4
    d = tiny(N=N, H=H, C=C, seed=8, mask="random:2")
    perm = torch.from_numpy(np.random.default_rng(1).permutation(N))
    dp = dict(d)
    for n in ("k", "v"):
        dp[n] = d[n][:, perm]
    dp["bias"] = d["bias"][:, :, perm]
    dp["mask"] = d["mask"][perm]
    o0, l0 = oracle.fwd(*args(d), d["mask"], STARTING, lib=lib)
    o1, l1 = oracle.fwd(*args(dp), dp["mask"], STARTING, lib=lib)
    close(o1, o0, TOL, "permutation: out")
    close(l1, l0, TOL, "permutation: lse")
    g0 = oracle.bwd(*args(d), d["dout"], d["mask"], STARTING, lib=lib)
    g1 = oracle.bwd(*args(dp), d["dout"], dp["mask"], STARTING, lib=lib)
    p = perm.numpy()
    close(g1[0], g0[0], TOL, "permutation: dq")
    close(g1[1], g0[1][:, p], TOL, "permutation: dk")
    close(g1[2], g0[2][:, p], TOL, "permutation: dv")
    close(g1[3], g0[3], TOL, "permutation: dgate")
    close(g1[4], g0[4][:, :, p], TOL, "permutation: dbias")


def check_variant_identity(lib=None):
    """ending(X) = T(starting(T(X))): T swaps the two residue axes of the pair
    tensors and of the bias; the key mask and lse stay in the variant frame."""
    N, H, C = 6, 2, 4
    d = tiny(N=N, H=H, C=C, seed=13, bias_std=np.sqrt(2.0), mask="random:2")
    dt = dict(d)
    for n in ("q", "k", "v", "gate", "dout"):
        dt[n] = d[n].transpose(0, 1).contiguous()
    dt["bias"] = d["bias"].transpose(1, 2).contiguous()
    oe, le = oracle.fwd(*args(d), d["mask"], ENDING, lib=lib)
    os_, ls = oracle.fwd(*args(dt), d["mask"], STARTING, lib=lib)
    close(oe, os_, 0.0, "ending vs transposed starting: out")
    close(le, ls, 0.0, "ending vs transposed starting: lse")
    ge = oracle.bwd(*args(d), d["dout"], d["mask"], ENDING, lib=lib)
    gs = oracle.bwd(*args(dt), dt["dout"], d["mask"], STARTING, lib=lib)
    for name, a, b in zip(("dq", "dk", "dv", "dgate"), ge[:4], gs[:4]):
        close(a, b, 0.0, f"ending vs transposed starting: {name}")
    close(ge[4], gs[4].transpose(0, 2, 1), 0.0, "ending vs transposed starting: dbias")


def check_fully_masked_row(lib=None):
    N, H, C = 6, 2, 4
    d = tiny(N=N, H=H, C=C, seed=17)
    m = full_mask(N, seed=17, keep_prob=0.7, fully_masked_rows=(2,))
    m[:, 0] = 1
    m[2, :] = 0
    out, lse = oracle.fwd(*args(d), m, STARTING, lib=lib)
    assert np.all(out[2] == 0.0)
    assert np.all(np.isneginf(lse[2]))
    assert np.all(np.isfinite(lse[[0, 1, 3, 4, 5]]))
    dq, dk, dv, dg, db = oracle.bwd(*args(d), d["dout"], m, STARTING, lib=lib)
    for name, a in (("dq", dq), ("dk", dk), ("dv", dv), ("dgate", dg)):
        assert np.all(a[2] == 0.0), name
    others = [0, 1, 3, 4, 5]
    db_others = oracle.bwd(*args(d), d["dout"], m, STARTING, rows=others, lib=lib)[4]
    close(db, db_others, TOL, "fully masked row adds nothing to dbias")


def check_sampled_entry_points(lib=None):
    """Row subsets and dbias entries agree with the full computation."""
    N, H, C = 9, 2, 4
    for variant in (STARTING, ENDING):
        d = tiny(N=N, H=H, C=C, seed=31, mask="random:2")
        out, lse = oracle.fwd(*args(d), d["mask"], variant, lib=lib)
        rows = [7, 0, 4]
        o2, l2 = oracle.fwd(*args(d), d["mask"], variant, rows=rows, lib=lib)
        close(o2, out[rows], 0.0, "row subset out")
        close(l2, lse[rows], 0.0, "row subset lse")
        full = oracle.bwd(*args(d), d["dout"], d["mask"], variant, lib=lib)
        sub = oracle.bwd(*args(d), d["dout"], d["mask"], variant, rows=rows, lib=lib)
        for name, a, b in zip(("dq", "dk", "dv", "dgate"), sub[:4], full[:4]):
            close(a, b[rows], 0.0, f"row subset {name}")
        ent = [(0, 1, 2), (1, 8, 0), (1, 3, 3), (0, 0, 8)]
        vals = oracle.dbias_entries(*args(d), d["dout"], ent, d["mask"], variant, lib=lib)
        close(vals, np.array([full[4][e] for e in ent]), 1e-13, "dbias entries")


CHECKS = [
    ("library composition (starting)", lambda lib: check_library_composition(lib, STARTING)),
    ("library composition (ending)", lambda lib: check_library_composition(lib, ENDING)),
    ("finite differences (starting)", lambda lib: check_finite_differences(lib, STARTING)),
    ("finite differences (ending)", lambda lib: check_finite_differences(lib, ENDING, N=3)),
    ("explicit Jacobian (starting)", lambda lib: check_jacobian(lib, STARTING)),
    ("explicit Jacobian (ending)", lambda lib: check_jacobian(lib, ENDING)),
    ("probabilities", check_probabilities),
    ("closed forms", check_closed_forms),
    ("invariants", check_invariants),
    ("permutation", check_permutation),
    ("variant identity", check_variant_identity),
    ("fully masked row", check_fully_masked_row),
    ("sampled entry points", check_sampled_entry_points),
]


@pytest.mark.parametrize("name,check", CHECKS, ids=[c[0] for c in CHECKS])
def test_oracle_pin(name, check):
    check(None)


def test_library_composition_full_mask():
    """Per-row key masks (row stride N) against the library composition."""
    d = tiny(N=6, H=2, C=4, seed=23)
    m = full_mask(6, seed=23, keep_prob=0.6)
    m[:, 1] = 1  # no fully masked row (SDPA would give NaN there)
    for variant in (STARTING, ENDING):
        ref = torch_reference(d, m, variant)
        out, lse = oracle.fwd(*args(d), m, variant)
        got = (out, lse) + oracle.bwd(*args(d), d["dout"], m, variant)
        for name, a, b in zip(("out", "lse", "dq", "dk", "dv", "dgate", "dbias"), got, ref):
            close(a, b, 1e-11, name)


# ----------------------------------------------------------------------------
# mutants: each plausible mistake must fail at least one pin
# ----------------------------------------------------------------------------

MUTANTS = {
    "bias term dropped":
        ("+ (double)p->bias[bias_at(p, h, x, y)];", "+ 0.0 * (double)p->bias[bias_at(p, h, x, y)];"),
    "bias transposed":
        ("if (p->variant == 0) return ((int64_t)h * p->N + x) * p->N + y;",
         "if (p->variant == 0) return ((int64_t)h * p->N + y) * p->N + x;"),
    "scale missing in logits":
        ("double s = scale * dot +", "double s = dot +"),
    "mask ignored":
        ("if (!p->mask) return 1;", "return 1;"),
    "max not subtracted in lse":
        ("const double lse = m + log(z);", "const double lse = log(z);"),
    "ds sign flipped":
        ("const double ds = pxy * (dp - D[x]);", "const double ds = pxy * (dp + D[x]);"),
    "dk uses k instead of q":
        ("dky[c] += scale * ds * (double)qx[c];", "dky[c] += scale * ds * (double)ky[c];"),
    "dq scale missing":
        ("dqx[c] += scale * ds * (double)ky[c];", "dqx[c] += ds * (double)ky[c];"),
    "dv uses ds":
        ("dvy[c] += pxy * du[x * C + c];", "dvy[c] += ds * du[x * C + c];"),
    "dgate misses (1 - s)":
        ("dg[c] = (double)ox[c] * u[x * C + c] * s * (1.0 - s);",
         "dg[c] = (double)ox[c] * u[x * C + c] * s;"),
    "D from dout instead of du":
        ("d += du[x * C + c] * u[x * C + c];", "d += (double)ox[c] * u[x * C + c];"),
    "ending reads pair tensors untransposed":
        ("int64_t a = (p->variant == 0) ? r : x;", "int64_t a = r;"),
    "ending bias untransposed":
        ("return ((int64_t)h * p->N + y) * p->N + x;\n}",
         "return ((int64_t)h * p->N + x) * p->N + y;\n}"),
    "dbias entries use the wrong key":
        ("const int64_t y = (variant == 0) ? b : a;", "const int64_t y = (variant == 0) ? a : b;"),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_mutants_are_caught(mutant):
    src = open(oracle._SRC).read()
    old, new = MUTANTS[mutant]
    assert src.count(old) == 1, f"mutation anchor not unique/absent: {old!r}"
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        msrc = os.path.join(tmp, "mutant.c")
        with open(msrc, "w") as f:
            f.write(src.replace(old, new))
        lib = oracle.load_library(oracle.build(force=True, src=msrc,
                                               lib=os.path.join(tmp, "libmutant.so")))
        failed = []
        for name, check in CHECKS:
            try:
                check(lib)
            except AssertionError:
                failed.append(name)
        assert failed, f"mutant '{mutant}' passed every pin"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
