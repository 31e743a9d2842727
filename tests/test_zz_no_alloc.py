"""tri_attn_fwd_noalloc: the forward for callers that may not allocate device
memory (its scratch is a fixed device array inside the library) must give the
same results as tri_attn_fwd with a caller workspace.

Collected last on purpose, and self-contained, so it passes both alone in a
fresh process and after the rest of the suite (when the shared scratch array
already holds an earlier call's leftovers)."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import triangle_attention_b200 as ta
from tri_inputs import ENDING, STARTING, full_mask, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu

F32_REL, BF16_REL, BF16_OUT_ABS, LSE_ABS = 1e-5, 1e-2, 2e-2, 1e-3


def noalloc_fn():
    f = ta.lib().tri_attn_fwd_noalloc
    P = ctypes.c_void_p
    f.argtypes = [ctypes.POINTER(ta.Problem), P, P, P, P, P, P, P, P, P]
    f.restype = ctypes.c_int
    return f


def ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def call_noalloc(g, variant):
    N, _, H, _ = g["q"].shape
    prob = ta.problem(g["q"], g["mask"], variant)
    out = torch.full_like(g["q"], float("nan"))
    lse = torch.full((N, H, N), float("nan"), dtype=torch.float32, device=g["q"].device)
    rc = noalloc_fn()(ctypes.byref(prob), ptr(g["q"]), ptr(g["k"]), ptr(g["v"]), ptr(g["bias"]),
                      ptr(g["gate"]), ptr(g["mask"]), ptr(out), ptr(lse),
                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, ta.STATUS.get(rc, rc)
    torch.cuda.synchronize()
    return out, lse


def rel_l2(a, b):
    a = a.detach().double().cpu().numpy().ravel()
    b = b.detach().double().cpu().numpy().ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def cases():
    c = []
    c.append(("bf16 N=256 starting, random key mask", workload_inputs("n256_bf16"), STARTING))
    d = make_inputs(200, H=2, c=32, dtype="bf16", seed=12, bias_std=1.4)
    d["mask"] = full_mask(200, seed=12, keep_prob=0.75, fully_masked_rows=(0, 129))
    c.append(("bf16 N=200 ending, per-row mask", d, ENDING))
    c.append(("fp32 N=37 starting, key mask",
              make_inputs(37, H=2, c=16, dtype="f32", seed=4, mask="random:5"), STARTING))
    return c


@pytest.mark.parametrize("name,d,variant", cases(), ids=lambda x: x if isinstance(x, str) else "")
def test_noalloc_matches_workspace_forward(name, d, variant):
    g = {k: (v.cuda().contiguous() if torch.is_tensor(v) else v) for k, v in d.items()}
    ref_out, ref_lse = ta.fwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], variant)
    torch.cuda.synchronize()
    # the oracle's answer on the same inputs, for the parity part of the check
    o_out, o_lse = oracle.fwd(d["q"], d["k"], d["v"], d["bias"], d["gate"], d["mask"], variant)
    o_out, o_lse = torch.from_numpy(np.asarray(o_out)), torch.from_numpy(np.asarray(o_lse))
    f32 = g["q"].dtype == torch.float32
    for call in range(2):                       # two calls in a row share the scratch
        out, lse = call_noalloc(g, variant)
        # the same kernels on the same inputs: the results must be the very same
        # bits as the forward with a caller workspace (a stale mask-bit or
        # transposed-bias block left in the shared array would show here)
        assert torch.equal(out, ref_out), f"call {call}: out differs from tri_attn_fwd"
        fin = torch.isfinite(ref_lse)
        assert torch.equal(torch.isfinite(lse), fin), f"call {call}: lse -inf pattern differs"
        assert torch.equal(lse[fin], ref_lse[fin]), f"call {call}: lse differs from tri_attn_fwd"
        # and within the parity tolerances of the oracle
        out_v = (out if variant == STARTING else out.transpose(0, 1)).double().cpu()
        err = rel_l2(out_v, o_out)
        assert err <= (F32_REL if f32 else BF16_REL), f"call {call}: out rel-L2 {err:.2e}"
        if not f32:
            m = float((out_v - o_out.double()).abs().max())
            assert m <= BF16_OUT_ABS, f"call {call}: out max-abs {m:.2e}"
        ofin = torch.isfinite(o_lse)
        assert torch.equal(torch.isfinite(lse).cpu(), ofin), f"call {call}: oracle -inf pattern"
        m = float((lse.cpu()[ofin].double() - o_lse[ofin].double()).abs().max()) \
            if ofin.any() else 0.0
        assert m <= LSE_ABS, f"call {call}: lse max-abs vs oracle {m:.2e}"


def test_noalloc_rejects_problems_beyond_its_scratch():
    # ending node at N=2048, H=4 needs a 33.5 MB transposed bias copy
    prob = ta.Problem(2048, 4, 32, ta.BF16, ENDING, 0)
    need = ta.fwd_workspace_size(prob)
    assert need > 16 << 20
    fake = ctypes.c_void_p(1 << 12)
    rc = noalloc_fn()(ctypes.byref(prob), fake, fake, fake, fake, fake, None, fake, fake, None)
    assert rc == 3   # TRI_ATTN_ERR_WORKSPACE, nothing enqueued
