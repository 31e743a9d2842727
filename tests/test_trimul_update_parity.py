"""Parity of the full triangle multiplicative update (tri_mul_update_fwd /
tri_mul_update_bwd) with its fp64 oracle (oracle/trimul_oracle.py, pinned in
tests/test_trimul_update_oracle.py): y, dz and every parameter gradient, both
edge directions, several channel counts, a position count that is not a
multiple of the GEMM tiles, and bit-identical repeats.

Tolerance: rel-L2 2e-2 on every output. The CUDA path rounds every value it
hands from one step to the next to bf16 (x, the pre-activations, a, b, t, u, h
and y; in the backward dh, the pre-activation gradients, dt, da and db), each a
relative error of at most 2^-9; about ten such roundings lie on each path
through the computation, and they add in quadrature, which gives a few 1e-3
and leaves a margin for the contraction's and the LayerNorms' amplification."""

import ctypes

import numpy as np
import pytest
import torch

import triangle_attention_b200 as ta
from oracle import trimul_oracle as T
from tri_inputs import make_update_inputs

TOL = 2e-2


def rel_l2(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def to_dev(d):
    dev = torch.device("cuda:0")
    return d["z"].to(dev), {k: v.to(dev) for k, v in d["params"].items()}, d["dy"].to(dev)


def test_sizes_and_limits_on_the_host():
    """Problem checks return before any CUDA call (no GPU needed)."""
    lib = ta.lib()
    s, w = ctypes.c_size_t(0), ctypes.c_size_t(0)
    ok = ta.MulUpdateProblem(64, 128, 128, ta.OUTGOING, 1e-5)
    assert lib.tri_mul_update_sizes(ctypes.byref(ok), ctypes.byref(s), ctypes.byref(w)) == 0
    R = 64 * 64
    assert s.value >= R * (2 * 128 + 8 + 2 * 640 + 4 * 2 * 128 + 8 + 2 * 128)
    for bad, code in [(ta.MulUpdateProblem(60, 128, 128, 0, 1e-5), 2),
                      (ta.MulUpdateProblem(64, 96, 128, 0, 1e-5), 2),
                      (ta.MulUpdateProblem(64, 128, 32, 0, 1e-5), 2),
                      (ta.MulUpdateProblem(64, 128, 128, 3, 1e-5), 1),
                      (ta.MulUpdateProblem(64, 128, 128, 0, 0.0), 1),
                      (ta.MulUpdateProblem(-8, 128, 128, 0, 1e-5), 1)]:
        assert lib.tri_mul_update_sizes(ctypes.byref(bad), ctypes.byref(s),
                                        ctypes.byref(w)) == code


CASES = [(64, 128, 128, ta.OUTGOING), (64, 128, 128, ta.INCOMING), (40, 64, 128, ta.OUTGOING),
         (24, 192, 64, ta.INCOMING), (16, 256, 256, ta.OUTGOING)]


@pytest.mark.gpu
@pytest.mark.parametrize("N,cz,c,direction", CASES)
def test_update_matches_oracle(N, cz, c, direction):
    d = make_update_inputs(N, cz=cz, c=c, seed=N + cz + c + direction)
    z, params, dy = to_dev(d)
    y, saved = ta.mul_update_fwd(z, params, direction)
    dz, grads = ta.mul_update_bwd(z, params, saved, dy, direction)
    torch.cuda.synchronize()
    ref_y, _ = T.update_fwd(d["z"], d["params"], direction)
    ref = T.update_bwd(d["z"], d["params"], direction, d["dy"])
    errs = {"y": rel_l2(np64(y), ref_y), "dz": rel_l2(np64(dz), ref["dz"])}
    for n in ta.MUL_UPDATE_PARAMS:
        errs[n] = rel_l2(np64(grads[n]), ref[n])
    bad = {k: v for k, v in errs.items() if not v <= TOL}
    assert not bad, f"rel-L2 above {TOL}: {bad} (all: {errs})"


@pytest.mark.gpu
def test_update_repeats_bit_identical_and_autograd():
    d = make_update_inputs(48, cz=128, c=128, seed=5)
    z, params, dy = to_dev(d)
    y1, s1 = ta.mul_update_fwd(z, params, ta.INCOMING)
    g1 = ta.mul_update_bwd(z, params, s1, dy, ta.INCOMING)
    y2, s2 = ta.mul_update_fwd(z, params, ta.INCOMING)
    g2 = ta.mul_update_bwd(z, params, s2, dy, ta.INCOMING)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(g1[0].view(torch.int16), g2[0].view(torch.int16))
    for n in ta.MUL_UPDATE_PARAMS:
        assert torch.equal(g1[1][n], g2[1][n]), n
    # the autograd function gives the same values
    zz = z.clone().requires_grad_(True)
    pp = {k: v.clone().requires_grad_(True) for k, v in params.items()}
    out = ta.triangle_multiplicative_update(zz, pp, ta.INCOMING)
    out.backward(dy)
    assert torch.equal(out.view(torch.int16), y1.view(torch.int16))
    assert torch.equal(zz.grad.view(torch.int16), g1[0].view(torch.int16))
    for n in ta.MUL_UPDATE_PARAMS:
        assert torch.equal(pp[n].grad.float(), g1[1][n].to(pp[n].dtype).float()), n
