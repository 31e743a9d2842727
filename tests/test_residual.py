"""Rounding-residual compensation ("TurboPairFormer accelera fino a 1,73x
l'addestramento di OpenFold3 nei test", section "Accuratezza e
riproducibilita"): the forward saves what rounding its output to bf16 removed,
without changing the bf16 output; the backward uses it for D = sum_c dout*out
(and dgate). Against the fp64 oracle the gradients that depend on D (dq, dk,
dbias, dgate) get closer; dv does not depend on D and stays bit-identical."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import triangle_attention_b200 as ta
from helpers import np64, rel_l2, to_device, variant_frame
from tri_inputs import ENDING, STARTING, workload_inputs


def P(N=64, dtype=ta.BF16):
    return ta.Problem(N, 4, 32, dtype, ta.STARTING, 0)


def test_options_rejections_on_the_host():
    lib = ta.lib()
    fake = ctypes.c_void_p(4096)
    args = [fake] * 5 + [None] + [fake, fake]
    ws = (fake, 1 << 30, None)
    # the first-version options size is accepted (checks continue to the workspace)
    v1 = ta.LaunchOpts(2 * 4 + 2 * ctypes.sizeof(ctypes.c_void_p), 0, None, None, None)
    assert lib.tri_attn_fwd_ex(ctypes.byref(P()), *args, None, 0, None, ctypes.byref(v1)) == 3
    # too small a size, or flags set
    bad = ta.LaunchOpts(8, 0, None, None, None)
    assert lib.tri_attn_fwd_ex(ctypes.byref(P()), *args, *ws, ctypes.byref(bad)) == 1
    flags = ta.LaunchOpts(ctypes.sizeof(ta.LaunchOpts), 1, None, None, None)
    assert lib.tri_attn_fwd_ex(ctypes.byref(P()), *args, *ws, ctypes.byref(flags)) == 1
    # a misaligned residual, and a residual on the fp32 path
    mis = ta.LaunchOpts(ctypes.sizeof(ta.LaunchOpts), 0, None, None, ctypes.c_void_p(4100))
    assert lib.tri_attn_fwd_ex(ctypes.byref(P()), *args, *ws, ctypes.byref(mis)) == 1
    f32 = ta.LaunchOpts(ctypes.sizeof(ta.LaunchOpts), 0, None, None, fake)
    assert lib.tri_attn_fwd_ex(ctypes.byref(P(N=32, dtype=ta.F32)), *args, *ws,
                               ctypes.byref(f32)) == 2
    bargs = [fake] * 5 + [None] + [fake] * 8
    assert lib.tri_attn_bwd_ex(ctypes.byref(P(N=32, dtype=ta.F32)), *bargs, *ws,
                               ctypes.byref(f32)) == 2


def run(g, variant, residual):
    res = torch.empty_like(g["q"]) if residual else None
    out, lse = ta.fwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], variant,
                      residual=res)
    grads = ta.bwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], out, lse, g["dout"],
                   variant, residual=res)
    torch.cuda.synchronize()
    return (out, lse) + tuple(grads), res


@pytest.mark.gpu
@pytest.mark.parametrize("name,variant", [("n384_bf16", STARTING), ("n384_bf16", ENDING),
                                          ("n256_bf16", STARTING)])
def test_residual_compensation_lowers_gradient_error(name, variant):
    d = workload_inputs(name)
    g = to_device(d, "cuda:0")
    plain, _ = run(g, variant, False)
    comp, res = run(g, variant, True)
    # the bf16 output, lse and dv do not change
    for i in (0, 1, 4):
        assert torch.equal(plain[i], comp[i])
    # the residual is what rounding removed: |res| <= half an ulp of out
    o = plain[0].float()
    r = res.float()
    assert torch.all(r.abs() <= o.abs() * 2.0 ** -8 + 1e-30)
    args = (d["q"], d["k"], d["v"], d["bias"], d["gate"])
    ref = oracle.bwd(*args, d["dout"], d["mask"], variant)
    names = ("dq", "dk", "dv", "dgate", "dbias")
    errs = {}
    for n, ref_t, idx in zip(names, ref, (2, 3, 4, 6, 5)):
        def err(t):
            got = np64(t) if n == "dbias" else np64(variant_frame(t, variant))
            return rel_l2(got, ref_t)
        errs[n] = (err(plain[idx]), err(comp[idx]))
    print(name, variant, {n: (f"{a:.3e}", f"{b:.3e}", f"{100 * (1 - b / a):.0f}%")
                          for n, (a, b) in errs.items()})
    for n in ("dq", "dk", "dbias", "dgate"):
        a, b = errs[n]
        assert b < a, f"{n}: compensated error {b:.3e} not below {a:.3e}"
    assert errs["dv"][0] == errs["dv"][1]
