"""The oracles against worked examples derived by hand (tests/golden/
closed_forms.json; each entry carries its derivation). CPU only."""

import json
import math
import os

import numpy as np

import oracle

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")))


def _num(v):
    return {"ln3": math.log(3.0), "ln4": math.log(4.0)}.get(v, v) if isinstance(v, str) else v


def test_attention_worked_example():
    g = GOLDEN["attention"]
    N, H, c = g["N"], g["H"], g["c"]
    q = np.zeros((N, N, H, c), np.float32)
    k = np.asarray(g["k"], np.float32)
    v = np.zeros((N, N, H, c), np.float32)
    for r in range(N):
        for y in range(N):
            v[r, y, 0] = g["v_rows"][y]
    bias = np.asarray([[[_num(e) for e in row] for row in hb] for hb in g["bias"]], np.float32)
    gate = np.zeros((N, N, H, c), np.float32)
    out, lse = oracle.fwd(q, k, v, bias, gate, None, oracle.STARTING)
    want = np.asarray(g["out"])
    for r in range(N):
        # bias entries are float32 roundings of ln 3: the probabilities are exact to ~1e-7
        np.testing.assert_allclose(out[r, :, 0, :], want, rtol=0, atol=1e-6)
        np.testing.assert_allclose(lse[r, 0, :], _num(g["lse"]), rtol=0, atol=1e-6)


def test_triangle_multiplication_worked_example():
    g = GOLDEN["triangle_multiplication"]
    a = np.asarray(g["a"], np.float32)[None]
    b = np.asarray(g["b"], np.float32)[None]
    # integer products: exact in fp64
    np.testing.assert_array_equal(oracle.mul_fwd(a, b, oracle.OUTGOING)[0], g["outgoing"])
    np.testing.assert_array_equal(oracle.mul_fwd(a, b, oracle.INCOMING)[0], g["incoming"])


def test_layer_norm_worked_example():
    g = GOLDEN["layer_norm"]
    z = np.asarray([g["z"]])
    x, mean, rstd = oracle.layer_norm(z, np.ones(4), np.zeros(4), 0.0)
    np.testing.assert_allclose(x[0] * math.sqrt(5.0), g["x_times_sqrt5"], rtol=1e-14, atol=1e-14)
    assert abs(mean[0] - g["mean"]) < 1e-15
    assert abs(rstd[0] ** 2 - g["rstd_squared"]) < 1e-15
