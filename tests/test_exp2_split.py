"""The FMA-pipe exp2 behind TRI_ATTN_OPT_EXP2_SPLIT: Cody and Waite's range
reduction and a degree-4 minimax polynomial for 2^f on [-1/2, 1/2].

CPU: the coefficients in the kernel source are the ones the committed Remez
script derives, and their fp64 relative error stays under the stated bound.
GPU: the device evaluation against fp64 exp2 over the whole exponent range the
forward produces, the hardware ex2.approx beside it, and forward parity with
the option on (the oracle does not change: the method's result is the same)."""

import re

import numpy as np
import pytest
import torch

import triangle_attention_b200 as ta
from triangle_attention_b200.csrc import gen_exp2_poly as gen

PTX = __import__("os").path.join(__import__("os").path.dirname(ta.__file__), "csrc", "ptx.cuh")
BOUND = 2.7e-6


def kernel_coefficients():
    src = open(PTX).read()
    body = src[src.index("exp2_fma2"):]
    body = body[:body.index("\n}\n")]
    lits = re.findall(r"0x1\.[0-9a-f]+p-?\d+f", body)
    seen = []
    for lit in lits:                              # each literal appears twice (a pair)
        v = float.fromhex(lit[:-1])
        if not seen or seen[-1] != v:
            seen.append(v)
    return seen[::-1]                             # Horner order is c4 .. c0


def test_coefficients_are_the_remez_ones():
    c32, bound = gen.coefficients_f32()
    assert kernel_coefficients() == [float(v) for v in c32]
    assert bound < BOUND


def test_polynomial_error_in_fp64():
    c = np.array(kernel_coefficients(), dtype=np.float64)
    f = np.linspace(-0.5, 0.5, 400001)
    err = np.polyval(c[::-1], f) / np.exp2(f) - 1.0
    assert np.max(np.abs(err)) < BOUND
    # the error equioscillates: the minimax property (degree 4: six extrema)
    signs = np.sign(err[np.abs(err) > 0.9 * np.max(np.abs(err))])
    assert np.count_nonzero(np.diff(signs)) >= 5


@pytest.mark.gpu
def test_device_exp2_against_fp64():
    rng = np.random.default_rng(3)
    x = np.concatenate([np.linspace(-125.0, 126.0, 1 << 20),
                        rng.uniform(-30.0, 8.0, 1 << 18)]).astype(np.float32)
    y_fma, y_mufu = ta.check_exp2(torch.from_numpy(x).cuda())
    ref = np.exp2(x.astype(np.float64))
    rel_fma = np.abs(y_fma.cpu().numpy().astype(np.float64) / ref - 1.0)
    rel_mufu = np.abs(y_mufu.cpu().numpy().astype(np.float64) / ref - 1.0)
    # polynomial bound plus the rounding of four fp32 FMAs and the final scaling
    assert rel_fma.max() < BOUND + 6e-7, rel_fma.max()
    assert rel_mufu.max() < 1e-6, rel_mufu.max()
    # below the clamp the polynomial returns about 2^-125, the hardware ex2 0
    lo_fma, lo_mufu = ta.check_exp2(torch.tensor([-200.0, -1e30], device="cuda"))
    assert np.allclose(lo_fma.cpu().numpy(), 2.0 ** -125, rtol=1e-5)
    assert np.all(lo_mufu.cpu().numpy() == 0.0)


@pytest.mark.gpu
@pytest.mark.parametrize("name,variant_name", [("n384_bf16", "ending"), ("n256_bf16", "starting")])
def test_forward_parity_with_the_split(name, variant_name):
    import oracle
    from helpers import compare_rows, to_device
    from tri_inputs import ENDING, STARTING, workload_inputs

    variant = ENDING if variant_name == "ending" else STARTING
    d = workload_inputs(name)
    g = to_device(d, "cuda:0")
    opts = ta.launch_opts(exp2_split=True)
    out, lse = ta.fwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], variant, opts=opts)
    out2, lse2 = ta.fwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], variant,
                        opts=ta.launch_opts(exp2_split=True))
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    N = d["q"].shape[0]
    ref = oracle.fwd(d["q"], d["k"], d["v"], d["bias"], d["gate"], d["mask"], variant)
    compare_rows({"out": out, "lse": lse}, ref, None, np.arange(N), variant, "bf16")


def test_backward_rejects_the_split_on_the_host():
    import ctypes
    lib = ta.lib()
    fake = ctypes.c_void_p(4096)
    bargs = [fake] * 5 + [None] + [fake] * 8
    opts = ta.launch_opts(exp2_split=True)
    prob = ta.Problem(64, 2, 32, ta.BF16, ta.STARTING, 0)
    assert lib.tri_attn_bwd_ex(ctypes.byref(prob), *bargs, fake, 1 << 40, None,
                               ctypes.byref(opts)) == 1
