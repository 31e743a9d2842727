"""LayerNorm and projection kernels against the fp64 oracle: every output
element at sizes spanning several 128-row tiles with ragged tails, every
supported channel count, a batch dimension, the empty problem; the full
N = 768 block on sampled rows (row-local outputs) and on every parameter
gradient (the oracle summed over row chunks, which is exact since those
gradients are sums over rows); bit-identical repeats. Host-side argument checks
run without a GPU.

Tolerances: x is LayerNorm in fp32 rounded once to bf16 (relative L2 about
2^-9/sqrt(3) = 1.1e-3); the projections and the bias read that rounded x and
round once more (about 2e-3); dz rounds an fp32 result once; the parameter
gradients are fp32 sums of products of bf16 values (x rounded). Bounds: 4e-3
on x, 8e-3 on the projected tensors, 1e-2 on every gradient, 1e-4 relative on
the fp32 statistics and on the column sums of exact bf16 values."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import triangle_attention_b200 as ta
from helpers import rel_l2
from tri_inputs import make_block_inputs

X_REL, PROJ_REL, GRAD_REL, F32_REL = 4e-3, 8e-3, 1e-2, 1e-4
EPS = 1e-5

# (N, cz, H, c, batch): ragged row tiles, every cz, H*c from 64 to 256
CASES = [(24, 128, 4, 32, None), (20, 64, 2, 32, 2), (17, 192, 3, 64, None),
         (12, 256, 8, 32, 3)]


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check(name, got, ref, rel):
    got = np64(got) if torch.is_tensor(got) else got
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    err = rel_l2(got, ref)
    assert err <= rel, f"{name}: relative L2 error {err:.3e} > {rel:.1e}"
    return err


def rows2d(t, cols):
    return t.reshape(-1, cols)


def bias_rows(t, H):
    """[.., H, N, N] -> [H][all rows] in the row order of the pair tensors."""
    b = t if t.dim() == 4 else t[None]
    return b.permute(1, 0, 2, 3).reshape(H, -1)


def to_dev(d, dev):
    return {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in d.items()}


# ------------------------------------------------------------- host checks --

def test_host_rejections():
    lib = ta.lib()
    fake = ctypes.c_void_p(4096)
    n = ctypes.c_size_t(0)
    good = ta.ProjProblem(64, 1, 128, 4, 32, 1e-5, 0)
    assert lib.tri_proj_workspace_size(ctypes.byref(good), ctypes.byref(n)) == 0
    need = n.value
    assert need >= 64 * 128 * 4
    bad = [(ta.ProjProblem(-1, 1, 128, 4, 32, 1e-5, 0), 1), (ta.ProjProblem(64, -1, 128, 4, 32, 1e-5, 0), 1),
           (ta.ProjProblem(64, 1, 128, 4, 32, 0.0, 0), 1), (ta.ProjProblem(64, 1, 128, 4, 32, 1e-5, 7), 1),
           (ta.ProjProblem(64, 1, 96, 4, 32, 1e-5, 0), 2), (ta.ProjProblem(64, 1, 320, 4, 32, 1e-5, 0), 2),
           (ta.ProjProblem(64, 1, 128, 9, 32, 1e-5, 0), 2), (ta.ProjProblem(64, 1, 128, 3, 16, 1e-5, 0), 2),
           (ta.ProjProblem(64, 1, 128, 8, 64, 1e-5, 0), 2),
           (ta.ProjProblem(1 << 20, 1 << 12, 128, 4, 32, 1e-5, 0), 2)]
    for prob, code in bad:
        assert lib.tri_proj_workspace_size(ctypes.byref(prob), ctypes.byref(n)) == code
        assert lib.tri_proj_out_fwd(ctypes.byref(prob), fake, fake, fake, fake, fake, 1 << 30,
                                    None) == code
    g = ctypes.byref(good)
    assert lib.tri_proj_in_fwd(g, *([fake] * 13), fake, need - 16, None) == 3
    assert lib.tri_proj_in_fwd(g, *([fake] * 13), None, need, None) == 3
    args = [fake] * 13
    args[6] = ctypes.c_void_p(4098)                     # misaligned x
    assert lib.tri_proj_in_fwd(g, *args, fake, need, None) == 1
    args = [fake] * 17
    args[12] = None                                     # missing dgamma
    assert lib.tri_proj_in_bwd(g, *args, fake, need, None) == 1
    assert lib.tri_proj_out_bwd(g, fake, fake, fake, fake, fake, None, fake, need, None) == 1


def test_workspace_grows_with_rows():
    small = ta.proj_workspace_size(ta.ProjProblem(64, 1, 128, 4, 32, 1e-5, 0))
    big = ta.proj_workspace_size(ta.ProjProblem(768 * 768, 1, 128, 4, 32, 1e-5, 0))
    assert big >= 768 * 768 * 128 * 4 > small        # the fp32 dx of the backward


# -------------------------------------------------------------- GPU parity --

def run_in(d, dev):
    g = to_dev(d, dev)
    f = ta.proj_in_fwd(g["z"], g["gamma"], g["beta"], g["w_qkvg"], g["b_g"], g["w_b"], EPS)
    x, stats = f[0], f[1]
    b = ta.proj_in_bwd(g["z"], g["gamma"], g["w_qkvg"], g["w_b"], x, stats, g["dq"], g["dk"],
                       g["dv"], g["dg"], g["dbias"], EPS)
    return f, b


def run_out(d, o, dev):
    g = to_dev(d, dev)
    o = o.to(dev)
    y = ta.proj_out_fwd(o, g["w_o"], g["b_o"])
    return y, ta.proj_out_bwd(o, g["w_o"], g["dy"])


def oracle_in(d, rows=None):
    cz, H = d["z"].shape[-1], d["w_b"].shape[1]
    z = rows2d(d["z"], cz)
    dq, dk, dv, dg = (rows2d(d[k], d[k].shape[-1] * d[k].shape[-2]) for k in
                      ("dq", "dk", "dv", "dg"))
    dbias = bias_rows(d["dbias"], H)
    if rows is not None:
        z, dq, dk, dv, dg, dbias = z[rows], dq[rows], dk[rows], dv[rows], dg[rows], dbias[:, rows]
    f = oracle.proj_in_fwd(z, d["gamma"], d["beta"], d["w_qkvg"], d["b_g"], d["w_b"], EPS)
    b = oracle.proj_in_bwd(z, d["gamma"], d["beta"], d["w_qkvg"], d["w_b"], EPS, dq, dk, dv, dg,
                           dbias)
    return f, b


def compare_in(f, b, rf, rb, H, rows=None):
    x, stats, q, k, v, g, bias = f
    cz = x.shape[-1]
    hc = q.shape[-1] * q.shape[-2]
    sel = (lambda a: a) if rows is None else (lambda a: a[rows])
    check("x", sel(rows2d(x, cz).cpu()), rf["x"], X_REL)
    st = sel(np64(stats).reshape(-1, 2))
    check("mean", st[:, 0], rf["mean"], F32_REL)
    check("rstd", st[:, 1], rf["rstd"], F32_REL)
    for name, t in (("q", q), ("k", k), ("v", v), ("gate", g)):
        check(name, sel(rows2d(t, hc).cpu()), rf[name], PROJ_REL)
    br = bias_rows(bias, H).cpu()
    check("bias", br if rows is None else br[:, rows], rf["bias"], PROJ_REL)
    check("dz", sel(rows2d(b[0], cz).cpu()), rb["dz"], GRAD_REL)


@pytest.mark.gpu
@pytest.mark.parametrize("N,cz,H,c,batch", CASES)
def test_input_side_matches_oracle(cuda_device, N, cz, H, c, batch):
    d = make_block_inputs(N, cz, H, c, batch, seed=N + cz)
    f, b = run_in(d, cuda_device)
    torch.cuda.synchronize()
    rf, rb = oracle_in(d)
    compare_in(f, b, rf, rb, H)
    for i, name in enumerate(("dgamma", "dbeta", "dw_qkvg", "db_g", "dw_b")):
        check(name, b[i + 1], rb[name], F32_REL if name == "db_g" else GRAD_REL)


@pytest.mark.gpu
@pytest.mark.parametrize("N,cz,H,c,batch", CASES)
def test_output_side_matches_oracle(cuda_device, N, cz, H, c, batch):
    d = make_block_inputs(N, cz, H, c, batch, seed=3 * N + cz)
    o = d["dq"]                                    # any bf16 [.., N, N, H, c] tensor
    y, (do, dw_o, db_o) = run_out(d, o, cuda_device)
    torch.cuda.synchronize()
    hc = H * c
    ref_y = oracle.proj_out_fwd(rows2d(o, hc), d["w_o"], d["b_o"])
    ref = oracle.proj_out_bwd(rows2d(o, hc), d["w_o"], rows2d(d["dy"], cz))
    check("y", rows2d(y, cz).cpu(), ref_y, PROJ_REL)
    check("do", rows2d(do, hc).cpu(), ref["do"], GRAD_REL)
    check("dw_o", dw_o, ref["dw_o"], GRAD_REL)
    check("db_o", db_o, ref["db_o"], F32_REL)


@pytest.mark.gpu
def test_empty_problem_zeroes_parameter_gradients(cuda_device):
    d = to_dev(make_block_inputs(4, 128, 4, 32, batch=1), cuda_device)
    z0 = d["z"][:0]
    f32 = dict(dtype=torch.float32, device=cuda_device)
    grads = (torch.empty_like(z0), torch.full((128,), 7.0, **f32), torch.full((128,), 7.0, **f32),
             torch.full((128, 512), 7.0, **f32), torch.full((128,), 7.0, **f32),
             torch.full((128, 4), 7.0, **f32))
    empty = d["dq"][:0]
    ta.proj_in_bwd(z0, d["gamma"], d["w_qkvg"], d["w_b"], z0, empty, empty, empty, empty, empty,
                   d["dbias"][:0], EPS, grads=grads)
    dw_o, db_o = torch.full((128, 128), 7.0, **f32), torch.full((128,), 7.0, **f32)
    ta.proj_out_bwd(empty, d["w_o"], z0, grads=(empty, dw_o, db_o))
    outs = ta.proj_in_fwd(z0, d["gamma"], d["beta"], d["w_qkvg"], d["b_g"], d["w_b"], EPS)
    torch.cuda.synchronize()
    assert all(int((t != 0).sum()) == 0 for t in grads[1:] + (dw_o, db_o))
    assert all(t.numel() == 0 for t in outs)


@pytest.mark.gpu
def test_repeats_are_bit_identical(cuda_device):
    d = make_block_inputs(96, 128, 4, 32, batch=None, seed=5)
    a = run_in(d, cuda_device)
    b = run_in(d, cuda_device)
    ya, ga = run_out(d, d["dv"], cuda_device)
    yb, gb = run_out(d, d["dv"], cuda_device)
    torch.cuda.synchronize()
    for s, t in zip(a[0] + a[1] + (ya,) + ga, b[0] + b[1] + (yb,) + gb):
        assert torch.equal(s, t)


@pytest.mark.gpu
def test_n768_sampled_rows_and_every_parameter_gradient(cuda_device):
    """The bench's configuration: N = 768, cz = 128, H = 4, c = 32. Row-local
    outputs on 4096 sampled rows (and the last one); every parameter gradient
    in full, the oracle summed over chunks of rows in order."""
    N, cz, H, c = 768, 128, 4, 32
    d = make_block_inputs(N, cz, H, c, None, seed=768)
    f, b = run_in(d, cuda_device)
    y, (do, dw_o, db_o) = run_out(d, d["dk"], cuda_device)
    torch.cuda.synchronize()
    R = N * N
    rows = np.sort(np.random.default_rng(1).choice(R - 1, 4095, replace=False))
    rows = np.append(rows, R - 1)
    rf, rb = oracle_in(d, rows)
    compare_in(f, b, rf, rb, H, rows)
    acc = {}
    step = 1 << 16
    for r0 in range(0, R, step):
        _, part = oracle_in(d, np.arange(r0, min(R, r0 + step)))
        for name in ("dgamma", "dbeta", "dw_qkvg", "db_g", "dw_b"):
            acc[name] = acc.get(name, 0.0) + part[name]
    for i, name in enumerate(("dgamma", "dbeta", "dw_qkvg", "db_g", "dw_b")):
        check(name, b[i + 1], acc[name], F32_REL if name == "db_g" else GRAD_REL)
    hc = H * c
    o = rows2d(d["dk"], hc)
    dy = rows2d(d["dy"], cz)
    check("y", rows2d(y, cz).cpu()[rows], oracle.proj_out_fwd(o[rows], d["w_o"], d["b_o"]),
          PROJ_REL)
    check("do", rows2d(do, hc).cpu()[rows], oracle.proj_out_bwd(o[rows], d["w_o"], dy[rows])["do"],
          GRAD_REL)
    ref_dw, ref_db = 0.0, 0.0
    for r0 in range(0, R, step):
        part = oracle.proj_out_bwd(o[r0:r0 + step], d["w_o"], dy[r0:r0 + step])
        ref_dw, ref_db = ref_dw + part["dw_o"], ref_db + part["db_o"]
    check("dw_o", dw_o, ref_dw, GRAD_REL)
    check("db_o", db_o, ref_db, F32_REL)
