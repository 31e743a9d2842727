"""Pins of the fp64 oracle of the full triangle multiplicative update
(oracle/trimul_oracle.py), each against something other than the oracle
itself: the pinned C oracle of the contraction, the identity between the two
edge directions, a closed form, central finite differences and torch's fp64
autograd. Planted mistakes (mutants) must each fail one of them."""

import numpy as np
import pytest
import torch

import oracle
from oracle import trimul_oracle as T
from tri_inputs import make_update_inputs

OUT, IN = T.OUTGOING, T.INCOMING


def small(seed=3, N=6, cz=8, c=4):
    return make_update_inputs(N, cz=cz, c=c, seed=seed)


def p64(p):
    return {k: np.asarray(v.double().numpy(), dtype=np.float64) for k, v in p.items()}


# ------------------------------------------------------------ pin functions --

def contraction_error(direction, seed=5):
    """t of the update against the C oracle of the contraction (channel-major)."""
    d = small(seed, N=7, cz=8, c=5)
    _, k = T.update_fwd(d["z"], d["params"], direction)
    N, c = k["N"], k["c"]
    a = torch.tensor(k["a"].reshape(N, N, c).transpose(2, 0, 1).copy(), dtype=torch.float32)
    b = torch.tensor(k["b"].reshape(N, N, c).transpose(2, 0, 1).copy(), dtype=torch.float32)
    # the C oracle takes float32 values: compare with the fp64 sums of those values
    ref = oracle.mul_fwd(a, b, direction)                       # [c][N][N]
    a64, b64 = a.double().numpy(), b.double().numpy()
    got = T.contract(a64.transpose(1, 2, 0), b64.transpose(1, 2, 0), direction)
    return float(np.max(np.abs(got.transpose(2, 0, 1) - ref)))


def direction_identity_error(seed=7):
    """With the output gate constant (W_g = 0), incoming(z) = outgoing(z^T) at
    every position: a and b of z^T at (i, k) are those of z at (k, i)."""
    d = small(seed)
    p = {k: v.clone() for k, v in d["params"].items()}
    cz = d["z"].shape[2]
    p["w_in"][:, -cz:] = 0
    y_in, _ = T.update_fwd(d["z"], p, IN)
    y_out_t, _ = T.update_fwd(d["z"].transpose(0, 1).contiguous(), p, OUT)
    return float(np.max(np.abs(y_in - y_out_t)))


def closed_form_error(seed=9, eps=1e-5):
    """W_in = 0: every pre-activation is its bias, so a = sigmoid(b_ag) b_ap and
    b = sigmoid(b_bg) b_bp per channel, t = N a b at every position, and y =
    sigmoid(b_g) (LayerNorm_out(N a b) W_o + b_o) at every position."""
    d = small(seed, N=5, cz=8, c=6)
    p = {k: v.clone() for k, v in d["params"].items()}
    p["w_in"].zero_()
    q = p64(p)
    N, cz, c = 5, 8, 6
    bi = q["b_in"]
    sig = lambda v: 1.0 / (1.0 + np.exp(-v))
    a = sig(bi[c:2 * c]) * bi[0:c]
    b = sig(bi[3 * c:4 * c]) * bi[2 * c:3 * c]
    t = N * a * b
    u = (t - t.mean()) / np.sqrt(((t - t.mean()) ** 2).mean() + eps) * q["ln_out_gamma"] \
        + q["ln_out_beta"]
    expect = sig(bi[4 * c:]) * (u @ q["w_o"] + q["b_o"])
    y, _ = T.update_fwd(d["z"], p, OUT, eps)
    return float(np.max(np.abs(y - expect[None, None, :])))


def finite_difference_error(direction, seed=11, h=1e-5):
    """Central differences of L = sum(dy y) against the oracle's gradients, on
    a handful of entries of z and of every parameter."""
    d = small(seed, N=4, cz=8, c=4)
    z = d["z"].double().numpy()
    p = p64(d["params"])
    dy = d["dy"].double().numpy()
    grads = T.update_bwd(z, p, direction, dy)
    rng = np.random.default_rng(seed)

    def loss(zz, pp):
        y, _ = T.update_fwd(zz, pp, direction)
        return float(np.sum(dy * y))

    worst = 0.0
    for name in ["z"] + sorted(p):
        arr = z if name == "z" else p[name]
        g = grads["dz"] if name == "z" else grads[name]
        for _ in range(4):
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            old = arr[idx]
            arr[idx] = old + h
            lp = loss(z, p)
            arr[idx] = old - h
            lm = loss(z, p)
            arr[idx] = old
            fd = (lp - lm) / (2 * h)
            worst = max(worst, abs(fd - g[idx]) / max(1.0, abs(fd)))
    return worst


def autograd_error(direction, seed=13, eps=1e-5):
    """The oracle's hand-written backward against torch's fp64 autograd of the
    same forward written with torch operations."""
    d = small(seed, N=5, cz=8, c=4)
    N, cz, c = 5, 8, 4
    z = d["z"].double().requires_grad_(True)
    p = {k: v.double().requires_grad_(True) for k, v in d["params"].items()}
    x = torch.nn.functional.layer_norm(z, (cz,), p["ln_gamma"], p["ln_beta"], eps)
    pre = x @ p["w_in"] + p["b_in"]
    a = torch.sigmoid(pre[..., c:2 * c]) * pre[..., 0:c]
    b = torch.sigmoid(pre[..., 3 * c:4 * c]) * pre[..., 2 * c:3 * c]
    t = torch.einsum("ikc,jkc->ijc", a, b) if direction == OUT else \
        torch.einsum("kic,kjc->ijc", a, b)
    u = torch.nn.functional.layer_norm(t, (c,), p["ln_out_gamma"], p["ln_out_beta"], eps)
    y = torch.sigmoid(pre[..., 4 * c:]) * (u @ p["w_o"] + p["b_o"])
    (y * d["dy"].double()).sum().backward()
    ref = T.update_bwd(d["z"], d["params"], direction, d["dy"])
    worst = float(np.max(np.abs(z.grad.numpy() - ref["dz"])))
    for k, v in p.items():
        worst = max(worst, float(np.max(np.abs(v.grad.numpy() - ref[k]))))
    return worst


# ---------------------------------------------------------------- the pins --

@pytest.mark.parametrize("direction", [OUT, IN])
def test_contraction_matches_the_c_oracle(direction):
    assert contraction_error(direction) < 1e-9


def test_incoming_is_outgoing_of_the_transposed_input():
    assert direction_identity_error() < 1e-12


def test_closed_form_with_zero_projections():
    assert closed_form_error() < 1e-12


@pytest.mark.parametrize("direction", [OUT, IN])
def test_backward_matches_finite_differences(direction):
    assert finite_difference_error(direction) < 1e-6


@pytest.mark.parametrize("direction", [OUT, IN])
def test_backward_matches_torch_autograd(direction):
    assert autograd_error(direction) < 1e-10


# ----------------------------------------------------------------- mutants --

def test_planted_mistakes_fail_a_pin(monkeypatch):
    """Each plausible mistake breaks at least one pin."""
    base_contract, base_sigmoid = T.contract, T._sigmoid
    base_ln_bwd = T.layer_norm_bwd
    # 1. the incoming sums taken as outgoing ones
    monkeypatch.setattr(T, "contract", lambda a, b, d: base_contract(a, b, OUT))
    assert contraction_error(IN) > 1e-6 or direction_identity_error() > 1e-6
    monkeypatch.setattr(T, "contract", base_contract)
    # 2. a and b swapped in the outgoing sum (t transposed)
    monkeypatch.setattr(T, "contract", lambda a, b, d: base_contract(b, a, d))
    assert contraction_error(OUT) > 1e-6
    monkeypatch.setattr(T, "contract", base_contract)
    # 3. a gate that is the logit itself (sigmoid dropped) in the forward
    monkeypatch.setattr(T, "_sigmoid", lambda v: v)
    assert closed_form_error() > 1e-6
    monkeypatch.setattr(T, "_sigmoid", base_sigmoid)
    # 4. the output LayerNorm's backward without its mean term
    def ln_bwd_no_mean(z, gamma, eps, dx):
        z = np.asarray(z, np.float64)
        mean = z.mean(axis=-1, keepdims=True)
        rstd = 1.0 / np.sqrt(((z - mean) ** 2).mean(axis=-1, keepdims=True) + eps)
        xhat = (z - mean) * rstd
        u = dx * np.asarray(gamma, np.float64)
        dz = rstd * (u - xhat * (u * xhat).mean(axis=-1, keepdims=True))
        return dz, (dx * xhat).sum(axis=0), dx.sum(axis=0)
    monkeypatch.setattr(T, "layer_norm_bwd", ln_bwd_no_mean)
    assert finite_difference_error(OUT) > 1e-4
    monkeypatch.setattr(T, "layer_norm_bwd", base_ln_bwd)
