"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before any CUDA call."""

import ctypes
import os
import re

import pytest
import torch

import triangle_attention_b200 as ta
from triangle_attention_b200 import build as tbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(tri_(?:attn|mul|proj)_\w+)\s*\(", src):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    tbuild.build()
    return ta.lib()


def test_header_declares_entry_points():
    names = declared_functions()
    for required in ("tri_attn_fwd", "tri_attn_bwd", "tri_attn_fwd_workspace_size",
                     "tri_attn_bwd_workspace_size", "tri_attn_read_status",
                     "tri_attn_status_string", "tri_attn_version", "tri_mul_fwd", "tri_mul_bwd",
                     "tri_proj_in_fwd", "tri_proj_in_bwd", "tri_proj_out_fwd",
                     "tri_proj_out_bwd", "tri_proj_workspace_size"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} is declared but not exported"


def test_version_and_status_strings(lib):
    assert lib.tri_attn_version() >> 16 == 1
    for code in range(7):
        assert lib.tri_attn_status_string(code).decode() == ta.STATUS[code]
    assert lib.tri_attn_status_string(99).decode() == "unknown status"


def P(N=64, H=4, c=32, dtype=ta.BF16, variant=ta.STARTING, stride=0):
    return ta.Problem(N, H, c, dtype, variant, stride)


def ws_size(lib, prob, which="fwd"):
    n = ctypes.c_size_t(0)
    f = lib.tri_attn_fwd_workspace_size if which == "fwd" else lib.tri_attn_bwd_workspace_size
    rc = f(ctypes.byref(prob), ctypes.byref(n))
    return rc, n.value


def test_workspace_sizes(lib):
    rc, n = ws_size(lib, P())
    assert rc == 0 and n >= 256
    rc, ne = ws_size(lib, P(variant=ta.ENDING))
    assert rc == 0 and ne >= n + 2 * 4 * 64 * 64       # transposed bias copy
    rc, nb = ws_size(lib, P(N=768), "bwd")
    assert rc == 0
    pair = 768 * 768 * 4 * 32
    # dU (bf16) + D + three sets of bf16 tile-contribution slots over 6 tiles
    assert nb >= 2 * pair + 4 * 768 * 768 * 4 + 3 * 6 * 2 * pair
    rc, nf = ws_size(lib, P(N=32, dtype=ta.F32), "bwd")
    assert rc == 0 and nf > 0


@pytest.mark.parametrize("prob,code", [
    (P(N=-1), 1), (P(H=0), 1), (P(c=0), 1), (P(dtype=7), 1), (P(variant=2), 1),
    (P(stride=5), 1), (P(c=65), 2), (P(dtype=ta.F32, c=65), 2),
])
def test_invalid_problems(lib, prob, code):
    rc, _ = ws_size(lib, prob)
    assert rc == code
    rc, _ = ws_size(lib, prob, "bwd")
    assert rc == code


@pytest.mark.parametrize("prob", [P(c=16), P(c=64), P(N=60), P(N=7, c=48), P(N=1)])
def test_bf16_shapes_of_the_cuda_core_kernels(lib, prob):
    """bf16 head dimensions other than 32 and N not a multiple of 8 run on the
    CUDA-core kernels: valid problems with a workspace of their own layout."""
    rc, n = ws_size(lib, prob)
    assert rc == 0 and n >= 4
    rc, nb = ws_size(lib, prob, "bwd")
    assert rc == 0 and nb > 0
    launches = ctypes.c_int32(0)
    assert lib.tri_attn_kernel_launches(ctypes.byref(prob), 0, 0, ctypes.byref(launches)) == 0
    assert launches.value == 1


def test_null_problem_and_null_size(lib):
    n = ctypes.c_size_t(0)
    assert lib.tri_attn_fwd_workspace_size(None, ctypes.byref(n)) == 1
    assert lib.tri_attn_fwd_workspace_size(ctypes.byref(P()), None) == 1


def test_host_side_rejections_before_any_launch(lib):
    """These return before any CUDA call, so they run without a GPU."""
    prob = P()
    fake = ctypes.c_void_p(4096)          # 256-aligned, never dereferenced
    z = None
    args = [fake] * 5 + [z] + [fake, fake]
    # missing workspace
    assert lib.tri_attn_fwd(ctypes.byref(prob), *args, z, 0, z) == 3
    # misaligned workspace
    assert lib.tri_attn_fwd(ctypes.byref(prob), *args, ctypes.c_void_p(4100), 1 << 20, z) == 3
    # too small a workspace
    assert lib.tri_attn_fwd(ctypes.byref(prob), *args, fake, 16, z) == 3
    # null and misaligned tensors
    bad = [fake] * 5 + [z] + [z, fake]
    assert lib.tri_attn_fwd(ctypes.byref(prob), *bad, fake, 1 << 30, z) == 1
    mis = [ctypes.c_void_p(4098)] + [fake] * 4 + [z] + [fake, fake]
    assert lib.tri_attn_fwd(ctypes.byref(prob), *mis, fake, 1 << 30, z) == 1
    # backward: invalid problem, then missing workspace
    bargs = [fake] * 5 + [z] + [fake] * 8
    assert lib.tri_attn_bwd(ctypes.byref(P(c=65)), *bargs, fake, 1 << 40, z) == 2
    assert lib.tri_attn_bwd(ctypes.byref(prob), *bargs, z, 0, z) == 3
    # N = 0 is a valid no-op
    zero = P(N=0)
    assert lib.tri_attn_fwd(ctypes.byref(zero), *args, fake, 1 << 20, z) == 0
    assert lib.tri_attn_bwd(ctypes.byref(zero), *bargs, fake, 1 << 20, z) == 0


def test_onchip_sum_option_on_the_host(lib):
    """TRI_ATTN_OPT_ONCHIP_SUMS: accepted by the bf16 backward only; the launch
    count and the workspace size cover that path. No CUDA call is made."""
    fake = ctypes.c_void_p(4096)
    z = None
    prob = P(N=768)
    args = [fake] * 5 + [z] + [fake, fake]
    bargs = [fake] * 5 + [z] + [fake] * 8
    opts = ta.launch_opts(onchip_sums=True)
    assert opts.flags == ta.OPT_ONCHIP_SUMS == 1
    # the forward takes no flags, and no flag but bit 0 exists
    assert lib.tri_attn_fwd_ex(ctypes.byref(prob), *args, fake, 1 << 40, z,
                               ctypes.byref(opts)) == 1
    bad = ta.launch_opts()
    bad.flags = 2
    assert lib.tri_attn_bwd_ex(ctypes.byref(prob), *bargs, fake, 1 << 40, z,
                               ctypes.byref(bad)) == 1
    # the fp32 backward rejects the bit
    f32 = P(N=32, dtype=ta.F32)
    assert lib.tri_attn_bwd_ex(ctypes.byref(f32), *bargs, fake, 1 << 40, z,
                               ctypes.byref(opts)) == 1
    # too small a workspace is still caught first
    assert lib.tri_attn_bwd_ex(ctypes.byref(prob), *bargs, fake, 16, z, ctypes.byref(opts)) == 3
    # launches: mask bits, preprocessing, one main launch for all 4 heads of
    # N=768 on 148 SMs (36 CTAs per head); the default path has 4
    n = ctypes.c_int32(0)
    assert lib.tri_attn_kernel_launches(ctypes.byref(prob), 2, 0, ctypes.byref(n)) == 0
    assert n.value == 3
    assert lib.tri_attn_kernel_launches(ctypes.byref(prob), 1, 0, ctypes.byref(n)) == 0
    assert n.value == 4
    assert lib.tri_attn_kernel_launches(ctypes.byref(prob), 3, 0, ctypes.byref(n)) == 1
    # the workspace holds the exchange ring of that path too: 8 slots x 4 pairs x
    # 3 kinds x 36 blocks of 128 x 32 bf16, plus dU and the (lse, D) pairs
    rc, nb = ws_size(lib, prob, "bwd")
    assert rc == 0
    pair = 768 * 768 * 4 * 32
    assert nb >= 2 * pair + 8 * 768 * 768 * 4 + 8 * 4 * 3 * 36 * 128 * 32 * 2


def test_batch_on_the_host(lib):
    """The batch field: validation, workspace growth, the calls that take one
    problem only, and launch counts (no CUDA call is made)."""
    def B(batch, reserved=0, **kw):
        p = P(**kw)
        p.batch, p.reserved = batch, reserved
        return p
    assert ws_size(lib, B(-1))[0] == 1
    assert ws_size(lib, B(2, reserved=1))[0] == 1
    assert ws_size(lib, B(65, N=1024))[0] == 1           # B*N above the N limit
    assert ws_size(lib, B(64, N=1024))[0] == 0
    # batch 0 and 1 are the same problem
    assert ws_size(lib, B(0)) == ws_size(lib, B(1))
    # an ending-node batch holds a transposed bias per problem
    rc1, n1 = ws_size(lib, B(1, variant=ta.ENDING))
    rc3, n3 = ws_size(lib, B(3, variant=ta.ENDING))
    assert rc1 == rc3 == 0 and n3 - n1 >= 2 * 2 * 4 * 64 * 64
    # the backward's scratch (dU, D, tile contributions) grows with the batch
    rc, nb1 = ws_size(lib, B(1, N=256), "bwd")
    rc, nb3 = ws_size(lib, B(3, N=256), "bwd")
    pair = 256 * 256 * 4 * 32
    assert nb3 - nb1 >= 2 * (2 * pair + 4 * 256 * 256 * 4 + 3 * 2 * 2 * pair)
    # row shards take one problem only
    fake = ctypes.c_void_p(4096)
    z = None
    prob = B(2)
    assert lib.tri_attn_fwd_rows(ctypes.byref(prob), 0, 8, *([fake] * 5), z, fake, fake, fake,
                                 ctypes.c_size_t(1 << 40), z) == 2
    assert lib.tri_attn_bwd_rows(ctypes.byref(prob), 0, 8, *([fake] * 5), z, *([fake] * 9),
                                 ctypes.c_size_t(1 << 40), z) == 2
    # launches: the tensor-core path runs a batch in one problem's launches; the
    # CUDA-core kernels take the problems in turn; the on-chip-sum option falls
    # back to the default backward for a batch
    n = ctypes.c_int32(0)
    for bwd in (0, 1):
        assert lib.tri_attn_kernel_launches(ctypes.byref(B(3)), bwd, 0, ctypes.byref(n)) == 0
        tc = n.value
        assert lib.tri_attn_kernel_launches(ctypes.byref(B(1)), bwd, 0, ctypes.byref(n)) == 0
        assert n.value == tc
    assert lib.tri_attn_kernel_launches(ctypes.byref(B(3, c=16)), 0, 0, ctypes.byref(n)) == 0
    assert n.value == 3
    assert lib.tri_attn_kernel_launches(ctypes.byref(B(2, N=768)), 2, 0, ctypes.byref(n)) == 0
    assert n.value == 4


def test_problem_of_batched_tensors():
    q = torch.empty((3, 16, 16, 2, 32), dtype=torch.bfloat16)
    p = ta.problem(q, torch.ones((3, 16), dtype=torch.uint8), ta.STARTING)
    assert (p.N, p.H, p.c, p.batch, p.mask_row_stride) == (16, 2, 32, 3, 0)
    p = ta.problem(q, torch.ones((3, 16, 16), dtype=torch.uint8), ta.ENDING)
    assert (p.batch, p.mask_row_stride) == (3, 16)
    assert ta.problem(q[0], None, ta.STARTING).batch == 1
    with pytest.raises(ValueError):
        ta.problem(q, torch.ones((2, 16), dtype=torch.uint8), ta.STARTING)
    with pytest.raises(ValueError):
        ta.problem(q, torch.ones((16,), dtype=torch.uint8), ta.STARTING)
    with pytest.raises(ValueError):
        ta.problem(torch.empty((3, 16, 15, 2, 32)), None, ta.STARTING)


def test_probe_mma_rejects_bad_arguments(lib):
    fake = ctypes.c_void_p(4096)
    for args in [(48, 0, 1, 1), (32, 3, 1, 1), (64, 1, 1, 1), (64, 2, 1, 1), (32, 0, 0, 1), (32, 0, 1, 0),
                 (32, 0, 2000, 1)]:
        assert lib.tri_attn_probe_mma(*args, fake, fake, None) == 1, args
    assert lib.tri_attn_probe_mma(32, 0, 1, 1, None, fake, None) == 1


def test_read_status_rejects_null(lib):
    v = ctypes.c_int32(0)
    assert lib.tri_attn_read_status(None, ctypes.byref(v), None) == 1
    assert lib.tri_attn_get_status(None, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(ta, "_lib", None)
    monkeypatch.setattr(ta, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        ta.lib()


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "triangle_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in src.lower().replace("oracle/", ""), f
