"""The differentiable entry points: torch.autograd through the CUDA path, with
and without a batch dimension; each batch element must give exactly what the
unbatched call gives, and the gradients must match the fp64 oracle."""

import numpy as np
import pytest
import torch

import oracle
import triangle_attention_b200 as ta
from helpers import BF16_REL, np64, rel_l2, to_device
from tri_inputs import STARTING, ENDING, make_inputs

pytestmark = pytest.mark.gpu


def batch_of(n, N, seed):
    ds = [make_inputs(N, H=2, c=32, dtype="bf16", seed=seed + i, mask="random:5") for i in range(n)]
    stack = {k: torch.stack([d[k] for d in ds]) for k in ("q", "k", "v", "bias", "gate", "dout",
                                                          "mask")}
    return ds, to_device(stack, "cuda:0")


@pytest.mark.parametrize("variant", [STARTING, ENDING])
def test_batched_attention_equals_unbatched_and_oracle(variant):
    ds, g = batch_of(3, 72, seed=40)
    leaves = {k: g[k].clone().requires_grad_(True) for k in ("q", "k", "v", "bias", "gate")}
    out = ta.triangle_attention(leaves["q"], leaves["k"], leaves["v"], leaves["bias"],
                                leaves["gate"], g["mask"], variant)
    out.backward(g["dout"])
    torch.cuda.synchronize()
    for i, d in enumerate(ds):
        gi = to_device(d, "cuda:0")
        o1, l1 = ta.fwd(gi["q"], gi["k"], gi["v"], gi["bias"], gi["gate"], gi["mask"], variant)
        grads = ta.bwd(gi["q"], gi["k"], gi["v"], gi["bias"], gi["gate"], gi["mask"], o1, l1,
                       gi["dout"], variant)
        assert torch.equal(out[i], o1)
        for name, ref in zip(("q", "k", "v", "bias", "gate"), grads[:3] + (grads[3], grads[4])):
            assert torch.equal(leaves[name].grad[i], ref), name
    # and the first element against the oracle
    d = ds[0]
    args = (d["q"], d["k"], d["v"], d["bias"], d["gate"])
    ref = oracle.bwd(*args, d["dout"], d["mask"], variant)
    got = leaves["bias"].grad[0]
    assert rel_l2(np64(got), ref[4]) <= BF16_REL


def test_triangle_multiplication_autograd():
    rng = np.random.default_rng(5)
    a, b, dt = (torch.from_numpy(rng.standard_normal((2, 4, 64, 64)).astype(np.float32))
                .to(torch.bfloat16).cuda() for _ in range(3))
    for direction in (ta.OUTGOING, ta.INCOMING):
        la, lb = a.clone().requires_grad_(True), b.clone().requires_grad_(True)
        t = ta.TriangleMultiplication.apply(la, lb, direction)
        t.backward(dt)
        torch.cuda.synchronize()
        for i in range(2):
            ref_t = oracle.mul_fwd(a[i].cpu(), b[i].cpu(), direction)
            ref_da, ref_db = oracle.mul_bwd(a[i].cpu(), b[i].cpu(), dt[i].cpu(), direction)
            assert rel_l2(np64(t[i]), ref_t) <= 4e-3
            assert rel_l2(np64(la.grad[i]), ref_da) <= 4e-3
            assert rel_l2(np64(lb.grad[i]), ref_db) <= 4e-3


@pytest.mark.parametrize("variant", [STARTING, ENDING])
def test_attention_block_matches_the_oracle_chain(variant):
    """LayerNorm -> projections -> attention -> output projection through
    autograd, against the oracles chained in fp64. Each GPU step rounds its
    outputs to bf16, so the bound is twice the single-kernel one."""
    from tri_inputs import full_mask, make_block_inputs
    N, cz, H, c, eps = 40, 128, 4, 32, 1e-5
    R, hc, shape = N * N, H * c, (N, N, H, c)
    d = make_block_inputs(N, cz, H, c, None, seed=50 + variant)
    mask = full_mask(N, seed=9, keep_prob=0.9)
    names = ("z", "gamma", "beta", "w_qkvg", "b_g", "w_b", "w_o", "b_o")
    leaves = {k: d[k].cuda().requires_grad_(True) for k in names}
    y = ta.triangle_attention_block(*(leaves[k] for k in names), mask.cuda(), variant, eps)
    y.backward(d["dy"].cuda())
    torch.cuda.synchronize()

    f = oracle.proj_in_fwd(d["z"].reshape(R, cz), d["gamma"], d["beta"], d["w_qkvg"], d["b_g"],
                           d["w_b"], eps)
    q, k, v, gate = (f[n].reshape(shape) for n in ("q", "k", "v", "gate"))
    bias = f["bias"].reshape(H, N, N)
    out, _ = oracle.fwd(q, k, v, bias, gate, mask, variant)
    out = oracle.to_storage(out, variant).reshape(R, hc)
    y_ref = oracle.proj_out_fwd(out, d["w_o"], d["b_o"])
    ob = oracle.proj_out_bwd(out, d["w_o"], d["dy"].reshape(R, cz))
    dq, dk, dv, dg, db = oracle.bwd(q, k, v, bias, gate, ob["do"].reshape(shape), mask, variant)
    dq, dk, dv, dg = (oracle.to_storage(t, variant).reshape(R, hc) for t in (dq, dk, dv, dg))
    ib = oracle.proj_in_bwd(d["z"].reshape(R, cz), d["gamma"], d["beta"], d["w_qkvg"], d["w_b"],
                            eps, dq, dk, dv, dg, db.reshape(H, R))
    tol = 2 * BF16_REL
    assert rel_l2(np64(y).reshape(R, cz), y_ref) <= tol
    ref = {"z": ib["dz"], "gamma": ib["dgamma"], "beta": ib["dbeta"], "w_qkvg": ib["dw_qkvg"],
           "b_g": ib["db_g"], "w_b": ib["dw_b"], "w_o": ob["dw_o"], "b_o": ob["db_o"]}
    for k in names:
        err = rel_l2(np64(leaves[k].grad).reshape(ref[k].shape), ref[k])
        assert err <= tol, f"d{k}: relative L2 error {err:.3e}"
