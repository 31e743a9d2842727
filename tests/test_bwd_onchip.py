"""Parity of the bf16 backward with on-chip tile sums (TRI_ATTN_OPT_ONCHIP_SUMS)
with the fp64 oracle, on the cases of the default path: every output element up
to N=384 (one, two and three tiles per axis, ragged tiles, shared and per-row
masks with fully masked rows, both variants, several row groups per head), and
at N=768 the attention rows on both sides of every tile boundary plus sampled
dbias entries. Repeated calls are bit-identical, and the results agree with the
default path's to the bf16 tolerance."""

import numpy as np
import pytest
import torch

import oracle
import triangle_attention_b200 as ta
from helpers import BF16_REL, assert_close, compare_rows, np64, to_device
from tri_inputs import ENDING, STARTING, full_mask, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dbias", "dgate")


def run(d, variant, onchip=True):
    g = to_device(d, "cuda:0")
    out, lse = ta.fwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], variant)
    opts = ta.launch_opts(onchip_sums=onchip)
    grads = ta.bwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], out, lse, g["dout"],
                   variant, opts=opts)
    torch.cuda.synchronize()
    res = dict(zip(GRADS, grads))
    res.update(out=out, lse=lse)
    return res


def check_against_oracle(d, variant, rows=None, n_entries=64):
    res = run(d, variant)
    N, _, H, _ = d["q"].shape
    rows = np.arange(N) if rows is None else np.asarray(rows)
    args = (d["q"], d["k"], d["v"], d["bias"], d["gate"])
    ref_f = oracle.fwd(*args, d["mask"], variant, rows=rows)
    ref_b = oracle.bwd(*args, d["dout"], d["mask"], variant, rows=rows)
    compare_rows(res, ref_f, ref_b, rows, variant, "bf16")
    if len(rows) == N:
        assert_close("dbias", np64(res["dbias"]), ref_b[4], BF16_REL)
    else:
        rng = np.random.default_rng(1)
        ent = np.stack([rng.integers(0, H, n_entries), rng.integers(0, N, n_entries),
                        rng.integers(0, N, n_entries)], axis=1)
        ref_db = oracle.dbias_entries(*args, d["dout"], ent, d["mask"], variant)
        db = np64(res["dbias"])[ent[:, 0], ent[:, 1], ent[:, 2]]
        assert_close("dbias (sampled)", db, ref_db, BF16_REL)
    return res


def per_row_mask_inputs():
    d = make_inputs(200, H=2, c=32, dtype="bf16", seed=12, bias_std=1.4)
    d["mask"] = full_mask(200, seed=12, keep_prob=0.75, fully_masked_rows=(0, 129))
    return d


@pytest.mark.parametrize("case", [
    "n8", "n136_key_mask", "n256_workload", "n200_row_mask", "n200_row_mask_ending",
    "n384_ending",
])
def test_full_parity(case):
    if case == "n8":
        check_against_oracle(make_inputs(8, H=2, c=32, dtype="bf16", seed=1), STARTING)
    elif case == "n136_key_mask":
        check_against_oracle(make_inputs(136, H=2, c=32, dtype="bf16", seed=1,
                                         mask="random:9"), STARTING)
    elif case == "n256_workload":
        check_against_oracle(workload_inputs("n256_bf16"), STARTING)
    elif case == "n200_row_mask":
        check_against_oracle(per_row_mask_inputs(), STARTING)
    elif case == "n200_row_mask_ending":
        check_against_oracle(per_row_mask_inputs(), ENDING)
    else:
        check_against_oracle(workload_inputs("n384_bf16"), ENDING)


def test_n768_tile_boundary_rows():
    """The full-size configuration: rows on both sides of each 128-tile edge."""
    rows = [0, 127, 128, 255, 256, 383, 384, 511, 512, 639, 640, 767]
    check_against_oracle(workload_inputs("n768_bf16"), STARTING, rows=rows)


@pytest.mark.parametrize("name,variant", [("n768_bf16", STARTING), ("n384_bf16", ENDING)])
def test_bit_identical_and_close_to_default_path(name, variant):
    d = workload_inputs(name)
    a = run(d, variant)
    b = run(d, variant)
    for n in GRADS:
        assert torch.equal(a[n].view(torch.int16), b[n].view(torch.int16)), f"{n} differs"
    base = run(d, variant, onchip=False)
    for n in GRADS:
        assert_close(n, np64(a[n]), np64(base[n]), BF16_REL)


def test_status_clean_and_launch_count():
    d = make_inputs(264, H=3, c=32, dtype="bf16", seed=5, mask="random:7")
    g = to_device(d, "cuda:0")
    out, lse = ta.fwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], STARTING)
    prob = ta.problem(g["q"], g["mask"], STARTING)
    ws = ta.workspace(ta.bwd_workspace_size(prob), g["q"].device)
    ta.bwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], out, lse, g["dout"],
           STARTING, ws=ws, opts=ta.launch_opts(onchip_sums=True))
    assert ta.read_status(ws) == 0
    assert ta.kernel_launches(prob, True, True, onchip_sums=True) >= 3
