"""Triangle-multiplication kernels against the fp64 oracle: every output
element, both edge directions, forward and backward, at sizes that span
several 128 x 128 tiles and 64-wide K slices with ragged tails; bit-identical
repeats. Host-side argument checks run without a GPU."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import triangle_attention_b200 as ta
from helpers import rel_l2

# bf16 inputs are exact, products accumulate in fp32 on the tensor cores and the
# result is rounded once to bf16: relative L2 error ~ 2^-9 / sqrt(3) ~ 1.1e-3.
MUL_REL = 4e-3


def stacks(C, N, seed):
    rng = np.random.default_rng(seed)
    return [torch.from_numpy(rng.standard_normal((C, N, N)).astype(np.float32)).to(torch.bfloat16)
            for _ in range(3)]


def test_host_rejections():
    lib = ta.lib()
    fake = ctypes.c_void_p(4096)
    n = ctypes.c_size_t(0)
    assert lib.tri_mul_workspace_size(ctypes.byref(ta.MulProblem(64, 4, 0)), ctypes.byref(n)) == 0
    assert n.value >= 4
    for prob, code in ((ta.MulProblem(-8, 4, 0), 1), (ta.MulProblem(64, 0, 0), 1),
                       (ta.MulProblem(64, 4, 2), 1), (ta.MulProblem(60, 4, 0), 2)):
        assert lib.tri_mul_workspace_size(ctypes.byref(prob), ctypes.byref(n)) == code
        assert lib.tri_mul_fwd(ctypes.byref(prob), fake, fake, fake, fake, 256, None) == code
    ok = ta.MulProblem(64, 4, 0)
    assert lib.tri_mul_fwd(ctypes.byref(ok), fake, fake, fake, None, 0, None) == 3
    assert lib.tri_mul_fwd(ctypes.byref(ok), ctypes.c_void_p(4098), fake, fake, fake, 256,
                           None) == 1
    assert lib.tri_mul_bwd(ctypes.byref(ok), fake, fake, fake, None, fake, fake, 256, None) == 1
    # N = 0 returns before any CUDA call (the fake pointers are never touched)
    assert lib.tri_mul_fwd(ctypes.byref(ta.MulProblem(0, 4, 1)), fake, fake, fake, fake, 256,
                           None) == 0
    assert lib.tri_mul_bwd(ctypes.byref(ta.MulProblem(0, 4, 1)), fake, fake, fake, fake, fake,
                           fake, 256, None) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("C,N", [(4, 64), (3, 136), (2, 200), (8, 256), (1, 8), (1, 512), (2, 520)])
@pytest.mark.parametrize("direction", [ta.OUTGOING, ta.INCOMING])
def test_mul_matches_oracle(C, N, direction):
    a, b, dt = stacks(C, N, seed=N + C + direction)
    ga, gb, gdt = (x.cuda() for x in (a, b, dt))
    t = ta.mul_fwd(ga, gb, direction)
    da, db = ta.mul_bwd(ga, gb, gdt, direction)
    torch.cuda.synchronize()
    ref_t = oracle.mul_fwd(a, b, direction)
    ref_da, ref_db = oracle.mul_bwd(a, b, dt, direction)
    for name, got, ref in (("t", t, ref_t), ("da", da, ref_da), ("db", db, ref_db)):
        g = got.to("cpu", torch.float64).numpy()
        assert np.all(np.isfinite(g)), name
        err = rel_l2(g, ref)
        assert err <= MUL_REL, f"{name}: rel-L2 {err:.3e}"


@pytest.mark.gpu
def test_mul_repeats_are_bit_identical_and_status_clean():
    a, b, dt = (x.cuda() for x in stacks(16, 384, seed=3))
    ws = ta.workspace(256, a.device)
    ref = (ta.mul_fwd(a, b, ta.OUTGOING, ws=ws),) + ta.mul_bwd(a, b, dt, ta.OUTGOING, ws=ws)
    for _ in range(2):
        got = (ta.mul_fwd(a, b, ta.OUTGOING, ws=ws),) + ta.mul_bwd(a, b, dt, ta.OUTGOING, ws=ws)
        assert all(torch.equal(x, y) for x, y in zip(got, ref))
    assert ta.read_status(ws) == 0


@pytest.mark.gpu
def test_mul_large_sampled_against_oracle():
    """N=768, C=128 (the attention bench's crop): sampled channels checked in full."""
    C, N = 128, 768
    a, b, dt = stacks(C, N, seed=7)
    ga, gb, gdt = (x.cuda() for x in (a, b, dt))
    for direction in (ta.OUTGOING, ta.INCOMING):
        t = ta.mul_fwd(ga, gb, direction)
        da, db = ta.mul_bwd(ga, gb, gdt, direction)
        torch.cuda.synchronize()
        for c in (0, 77, 127):
            sl = slice(c, c + 1)
            ref_t = oracle.mul_fwd(a[sl], b[sl], direction)
            ref_da, ref_db = oracle.mul_bwd(a[sl], b[sl], dt[sl], direction)
            for name, got, ref in (("t", t, ref_t), ("da", da, ref_da), ("db", db, ref_db)):
                err = rel_l2(got[sl].to("cpu", torch.float64).numpy(), ref)
                assert err <= MUL_REL, f"{name} c={c} dir={direction}: {err:.3e}"
