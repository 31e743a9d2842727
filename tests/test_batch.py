"""Batches of independent problems [B, N, N, H, c] in one call: on the
tensor-core path the B problems share each kernel launch (attention row r of
problem b is row b*N + r of the launch), on the CUDA-core path they run one
after another. Every problem of a batch must give, bit for bit, what a call on
that problem alone gives, and one problem per case is checked against the fp64
oracle element by element."""

import numpy as np
import pytest
import torch

import oracle
import triangle_attention_b200 as ta
from helpers import compare_rows, run_cuda, to_device, assert_close, np64, BF16_REL, F32_REL
from tri_inputs import ENDING, STARTING, full_mask, make_inputs

pytestmark = pytest.mark.gpu

KEYS = ("q", "k", "v", "bias", "gate", "dout")
OUTS = ("out", "lse", "dq", "dk", "dv", "dbias", "dgate")


def draw_batch(B, N, H, c, dtype, mask, seed):
    ds = []
    for i in range(B):
        d = make_inputs(N, H=H, c=c, dtype=dtype, seed=seed + i,
                        mask="none" if mask == "rows" else mask)
        if mask == "rows":
            # per-row masks; problem 1 has a fully masked row
            d["mask"] = full_mask(N, seed=seed + i, keep_prob=0.75,
                                  fully_masked_rows=(5,) if i == 1 else ())
        ds.append(d)
    stack = {k: torch.stack([d[k] for d in ds]) for k in KEYS}
    stack["mask"] = None if ds[0]["mask"] is None else torch.stack([d["mask"] for d in ds])
    return ds, to_device(stack, "cuda:0")


def run_batched(g, variant):
    out, lse = ta.fwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], variant)
    dq, dk, dv, db, dg = ta.bwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], out, lse,
                                g["dout"], variant)
    torch.cuda.synchronize()
    return dict(out=out, lse=lse, dq=dq, dk=dk, dv=dv, dbias=db, dgate=dg)


@pytest.mark.parametrize("variant", [STARTING, ENDING], ids=["starting", "ending"])
@pytest.mark.parametrize("N,H,c,dtype,mask", [
    (136, 2, 32, "bf16", "random:9"),   # tensor cores, a ragged second tile, many row groups
    (72, 3, 32, "bf16", "rows"),        # per-row masks, a fully masked row in problem 1
    (256, 4, 32, "bf16", "none"),       # two full tiles, several row groups (dbias reduction)
    (40, 2, 16, "bf16", "random:3"),    # bf16 on the CUDA-core kernels
    (33, 2, 8, "f32", "random:3"),      # fp32
], ids=["tc_ragged", "tc_rowmask", "tc_n256", "core_bf16", "core_f32"])
def test_batch_equals_each_problem_alone_and_the_oracle(variant, N, H, c, dtype, mask):
    B = 3
    ds, g = draw_batch(B, N, H, c, dtype, mask, seed=100 + N)
    got = run_batched(g, variant)
    assert got["lse"].shape == (B, N, H, N)
    for i, d in enumerate(ds):
        alone = run_cuda(d, variant)
        for name in OUTS:
            assert torch.equal(got[name][i], alone[name]), f"problem {i}: {name}"
    # problem 1 against the oracle, every element
    d = ds[1]
    args = (d["q"], d["k"], d["v"], d["bias"], d["gate"])
    ref_f = oracle.fwd(*args, d["mask"], variant)
    ref_b = oracle.bwd(*args, d["dout"], d["mask"], variant)
    one = {k: got[k][1] for k in OUTS}
    compare_rows(one, ref_f, ref_b, np.arange(N), variant, dtype)
    assert_close("dbias", np64(one["dbias"]), ref_b[4], F32_REL if dtype == "f32" else BF16_REL)


def test_batch_with_one_row_group_writes_dbias_directly():
    """N=640, H=4: 100 tiles per problem, one row group, so the backward writes
    dbias from the main kernel; two problems in one launch, both variants."""
    ds, g = draw_batch(2, 640, 4, 32, "bf16", "random:40", seed=7)
    for variant in (STARTING, ENDING):
        got = run_batched(g, variant)
        for i, d in enumerate(ds):
            alone = run_cuda(d, variant)
            for name in OUTS:
                assert torch.equal(got[name][i], alone[name]), f"{variant} problem {i}: {name}"


def test_batch_launch_count_is_that_of_one_problem():
    """The tensor-core path runs a batch in the launches of one problem."""
    q = torch.empty((4, 64, 64, 2, 32), dtype=torch.bfloat16)
    for variant in (STARTING, ENDING):
        one = ta.problem(q[0], None, variant)
        many = ta.problem(q, None, variant)
        for bwd in (False, True):
            assert ta.kernel_launches(many, bwd, False) == ta.kernel_launches(one, bwd, False)


def test_calls_from_a_fresh_host_thread():
    """A host thread whose first CUDA work is a call into the library (so no
    context is current on it yet) gets the same results as the main thread."""
    import threading
    ds, g = draw_batch(2, 72, 2, 32, "bf16", "random:5", seed=40)
    ref = run_batched(g, STARTING)
    box = {}

    def work():
        try:
            box["res"] = run_batched(g, STARTING)
        except Exception as e:            # surfaced below, on the test's thread
            box["err"] = e

    t = threading.Thread(target=work)
    t.start()
    t.join()
    assert "err" not in box, box.get("err")
    for name in OUTS:
        assert torch.equal(box["res"][name], ref[name]), name


def test_onchip_option_with_a_batch_takes_the_default_backward():
    """TRI_ATTN_OPT_ONCHIP_SUMS applies to single problems; a batch takes the
    default backward and gives its bits."""
    ds, g = draw_batch(2, 136, 2, 32, "bf16", "random:9", seed=11)
    out, lse = ta.fwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], STARTING)
    args = (g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], out, lse, g["dout"], STARTING)
    plain = ta.bwd(*args)
    opt = ta.bwd(*args, opts=ta.launch_opts(onchip_sums=True))
    torch.cuda.synchronize()
    for a, b, name in zip(plain, opt, ("dq", "dk", "dv", "dbias", "dgate")):
        assert torch.equal(a, b), name


def test_exp2_split_forward_with_a_batch():
    """The forward with one exponential pair in four on the FMA pipe runs a batch
    in one launch too: each problem bit-identical to the same option alone."""
    ds, g = draw_batch(3, 72, 2, 32, "bf16", "rows", seed=13)
    opts = ta.launch_opts(exp2_split=True)
    out, lse = ta.fwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], ENDING, opts=opts)
    torch.cuda.synchronize()
    for i, d in enumerate(ds):
        gi = to_device(d, "cuda:0")
        o1, l1 = ta.fwd(gi["q"], gi["k"], gi["v"], gi["bias"], gi["gate"], gi["mask"], ENDING,
                        opts=ta.launch_opts(exp2_split=True))
        torch.cuda.synchronize()
        assert torch.equal(out[i], o1) and torch.equal(lse[i], l1), i
