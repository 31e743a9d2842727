"""Pins of the triangle-multiplication oracle (CPU, fp64). The pages give no
formula and no worked example, so the oracle is pinned to facts that hold for
the contraction independently of how it is coded: closed forms, the relation
between the two edge directions, the adjoint identity of a bilinear map and
exact finite differences; a mutation test checks that plausible mistakes in
the oracle's indices trip at least one pin."""

import os

import numpy as np
import pytest

import oracle

OUT, INC = oracle.OUTGOING, oracle.INCOMING


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def T(x):
    """swap the two residue axes of a channel-major stack"""
    return np.ascontiguousarray(np.swapaxes(x, 1, 2))


def pins(lib=None):
    """Every pin; returns the names of those that fail (empty = all hold)."""
    failed = []
    C, N = 3, 7
    a, b, dt = rand((C, N, N), 1), rand((C, N, N), 2), rand((C, N, N), 3)
    # closed form: all-ones inputs give N everywhere, both directions
    ones = np.ones((C, N, N), np.float32)
    for d in (OUT, INC):
        if not np.allclose(oracle.mul_fwd(ones, ones, d, lib=lib), N, rtol=0, atol=1e-12):
            failed.append(f"ones-{d}")
    # closed form: a one-hot in the summed index selects a slice of b
    k0 = 4
    hot = np.zeros((C, N, N), np.float32)
    hot[:, :, k0] = 1.0                                      # a[c][i][k] = [k == k0]
    if not np.array_equal(oracle.mul_fwd(hot, b, OUT, lib=lib), np.broadcast_to(
            b[:, None, :, k0], (C, N, N))):
        failed.append("onehot-out")
    if not np.array_equal(oracle.mul_fwd(T(hot), b, INC, lib=lib), np.broadcast_to(
            b[:, k0, None, :], (C, N, N))):
        failed.append("onehot-in")
    # the incoming direction is the outgoing one on residue-transposed inputs
    if not np.allclose(oracle.mul_fwd(a, b, INC, lib=lib), oracle.mul_fwd(T(a), T(b), OUT, lib=lib),
                       rtol=0, atol=1e-12):
        failed.append("direction-fwd")
    da_i, db_i = oracle.mul_bwd(a, b, dt, INC, lib=lib)
    da_o, db_o = oracle.mul_bwd(T(a), T(b), dt, OUT, lib=lib)
    if not (np.allclose(da_i, T(da_o), atol=1e-12) and np.allclose(db_i, T(db_o), atol=1e-12)):
        failed.append("direction-bwd")
    # adjoint identity of a bilinear map: <dt, t> = <da, a> = <db, b>
    for d in (OUT, INC):
        t = oracle.mul_fwd(a, b, d, lib=lib)
        da, db = oracle.mul_bwd(a, b, dt, d, lib=lib)
        L = float(np.sum(dt.astype(np.float64) * t))
        if not (np.isclose(L, np.sum(da * a), rtol=1e-12) and
                np.isclose(L, np.sum(db * b), rtol=1e-12)):
            failed.append(f"adjoint-{d}")
        # finite differences are exact for a linear map (up to rounding)
        rng = np.random.default_rng(9)
        h = 0.5
        for _ in range(6):
            c, r, s = rng.integers(0, C), rng.integers(0, N), rng.integers(0, N)
            for x, g, name in ((a, da, "a"), (b, db, "b")):
                xp, xm = x.copy(), x.copy()
                xp[c, r, s] += h
                xm[c, r, s] -= h
                args_p = (xp, b) if name == "a" else (a, xp)
                args_m = (xm, b) if name == "a" else (a, xm)
                # the actual float32 step (x + h rounds), so the quotient is exact
                step = float(xp[c, r, s]) - float(xm[c, r, s])
                fd = (np.sum(dt * oracle.mul_fwd(*args_p, d, lib=lib)) -
                      np.sum(dt * oracle.mul_fwd(*args_m, d, lib=lib))) / step
                if not np.isclose(fd, g[c, r, s], rtol=1e-9, atol=1e-9):
                    failed.append(f"fd-{name}-{d}")
                    break
    # N = 0 is empty, not an error
    if oracle.mul_fwd(np.zeros((2, 0, 0), np.float32), np.zeros((2, 0, 0), np.float32),
                      OUT, lib=lib).shape != (2, 0, 0):
        failed.append("empty")
    return failed


def test_oracle_meets_every_pin():
    assert pins() == []


def test_oracle_rejects_bad_direction():
    with pytest.raises(RuntimeError):
        oracle.mul_fwd(rand((1, 3, 3), 0), rand((1, 3, 3), 1), 2)


MUTANTS = {
    "outgoing reads b[k][j]": ("at(a, N, c, i, k) * at(b, N, c, j, k)",
                               "at(a, N, c, i, k) * at(b, N, c, k, j)"),
    "incoming reads a[i][k]": ("at(a, N, c, k, i) * at(b, N, c, k, j)",
                               "at(a, N, c, i, k) * at(b, N, c, k, j)"),
    "outgoing da reads b[k][j]": ("ga += at(dt, N, c, r, j) * at(b, N, c, j, s)",
                                  "ga += at(dt, N, c, r, j) * at(b, N, c, s, j)"),
    "outgoing db uses b": ("gb += at(dt, N, c, i, r) * at(a, N, c, i, s)",
                           "gb += at(dt, N, c, i, r) * at(b, N, c, i, s)"),
    "incoming da transposes dt": ("ga += at(dt, N, c, s, j) * at(b, N, c, r, j)",
                                  "ga += at(dt, N, c, j, s) * at(b, N, c, r, j)"),
    "incoming db reads a[i][k]": ("gb += at(dt, N, c, i, s) * at(a, N, c, r, i)",
                                  "gb += at(dt, N, c, i, s) * at(a, N, c, i, r)"),
    "sum skips the last k": ("for (int64_t k = 0; k < N; ++k)",
                             "for (int64_t k = 0; k + 1 < N; ++k)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_mutant_fails_a_pin(name, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "tri_mul_oracle.c")).read()
    old, new = MUTANTS[name]
    assert old in src, name
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    lib = oracle.load_mul_library(oracle.build(True, str(mut), str(tmp_path / "libmut.so")))
    assert pins(lib) != [], f"mutant '{name}' passes every pin"
