"""Row shards: one problem split by attention rows across ranks (the row-wise
split of the pair representation of "FastFold: Reducing AlphaFold Training
Time from 11 Days to 67 Hours", methods, Dynamic Axial Parallelism, applied to
this operation). Every rank computes its rows of out, lse, dq, dk, dv and dgate
and an fp32 partial of dbias; the partials are gathered and added in rank
order on the GPU.

CPU: the partition, the host-side argument checks of the shard calls, and the
rank-ordered gather over two gloo ranks. GPU: shards run one after another on
one GPU give, on every row, the same bits as the whole-problem call, and the
rank-ordered dbias matches the oracle."""

import ctypes
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import triangle_attention_b200 as ta
from triangle_attention_b200 import build as tbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# ------------------------------------------------------------------- CPU --

@pytest.mark.parametrize("N,world", [(8, 1), (264, 2), (264, 4), (768, 3), (768, 8), (1536, 5)])
def test_shard_rows_partition(N, world):
    shards = [ta.shard_rows(N, world, r) for r in range(world)]
    pos = 0
    for begin, count in shards:                  # contiguous, in rank order
        assert begin == pos and begin % 8 == 0 and count % 8 == 0
        pos += count
    assert pos == N
    counts = [c for _, c in shards]
    assert max(counts) - min(counts) <= 8        # balanced to one 8-row group


def test_shard_rows_rejects_bad_splits():
    with pytest.raises(ValueError):
        ta.shard_rows(260, 2, 0)                 # N not a multiple of 8
    with pytest.raises(ValueError):
        ta.shard_rows(264, 2, 2)                 # rank out of range


def test_shard_calls_rejected_on_host():
    """Argument errors return before any CUDA call (no GPU needed)."""
    tbuild.build()
    lib = ta.lib()
    fake = ctypes.c_void_p(4096)
    z = None
    P = lambda dtype=ta.BF16: ta.Problem(64, 2, 32, dtype, ta.STARTING, 0)
    fargs = [fake] * 5 + [z] + [fake, fake, fake, 1 << 30, z]
    bargs = [fake] * 5 + [z] + [fake] * 8 + [fake, 1 << 30, z]
    # a shard is whole 8-row groups inside [0, N)
    assert lib.tri_attn_fwd_rows(ctypes.byref(P()), 4, 8, *fargs) == 1
    assert lib.tri_attn_fwd_rows(ctypes.byref(P()), 0, 12, *fargs) == 1
    assert lib.tri_attn_fwd_rows(ctypes.byref(P()), 56, 16, *fargs) == 1
    assert lib.tri_attn_fwd_rows(ctypes.byref(P()), -8, 8, *fargs) == 1
    assert lib.tri_attn_bwd_rows(ctypes.byref(P()), 8, 4, *bargs) == 1
    # bf16 only
    assert lib.tri_attn_fwd_rows(ctypes.byref(P(ta.F32)), 0, 8, *fargs) == 2
    assert lib.tri_attn_bwd_rows(ctypes.byref(P(ta.F32)), 0, 8, *bargs) == 2
    # the backward needs its dbias partial
    nodb = [fake] * 5 + [z] + [fake] * 6 + [z, fake] + [fake, 1 << 30, z]
    assert lib.tri_attn_bwd_rows(ctypes.byref(P()), 0, 8, *nodb) == 1
    # an empty shard is a valid no-op
    assert lib.tri_attn_fwd_rows(ctypes.byref(P()), 64, 0, *fargs) == 0
    # the rank-ordered sum: count >= 1, aligned pointers
    assert lib.tri_attn_dbias_reduce(fake, 0, 64, 2, fake, z) == 1
    assert lib.tri_attn_dbias_reduce(ctypes.c_void_p(4100), 2, 64, 2, fake, z) == 1
    assert lib.tri_attn_dbias_reduce(z, 2, 64, 2, fake, z) == 1


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, world, port, queue):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    import triangle_attention_b200 as ta

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        begin, count = ta.shard_rows(264, world, rank)
        # a partial that tells the ranks apart and is not symmetric in them
        partial = torch.arange(3 * 5 * 5, dtype=torch.float32).reshape(3, 5, 5) * (rank + 1) \
            + 0.25 * rank
        stacked = ta.gather_partials(partial)
        queue.put((rank, begin, count, stacked.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gather_partials_in_rank_order():
    world = 2
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=rank_main, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        results = sorted((queue.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
        for p in procs:
            p.join(timeout=60)
        codes = [p.exitcode for p in procs]
    finally:
        for p in procs:
            if p.is_alive():
                p.kill()
    assert codes == [0, 0], f"rank exit codes {codes}"
    expect = [np.arange(75, dtype=np.float32).reshape(3, 5, 5) * (r + 1) + 0.25 * r
              for r in range(world)]
    for rank, begin, count, stacked in results:
        assert (begin, count) == ta.shard_rows(264, world, rank)
        assert stacked.shape == (world, 3, 5, 5)
        for r in range(world):               # every rank holds the same stack, rank order
            assert np.array_equal(stacked[r], expect[r])
    # the rows of the two ranks cover every row once
    covered = sorted(x for _, b, c, _ in results for x in range(b, b + c))
    assert covered == list(range(264))


# ------------------------------------------------------------------- GPU --

def _run_shards(g, variant, world):
    N = g["q"].shape[0]
    out = torch.full_like(g["q"], float("nan"))
    lse = torch.full((N, g["q"].shape[2], N), float("nan"), device=g["q"].device)
    for r in range(world):
        b, c = ta.shard_rows(N, world, r)
        ta.fwd_rows(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], variant, b, c,
                    out=out, lse=lse)
    grads = [torch.full_like(g["q"], float("nan")) for _ in range(3)]
    dgate = torch.full_like(g["gate"], float("nan"))
    partials = []
    for r in range(world):
        b, c = ta.shard_rows(N, world, r)
        dbp = torch.empty(g["bias"].shape, dtype=torch.float32, device=g["q"].device)
        ta.bwd_rows(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], out, lse, g["dout"],
                    variant, b, c, grads=(grads[0], grads[1], grads[2], dbp, dgate))
        partials.append(dbp)
    dbias = ta.dbias_reduce(torch.stack(partials))
    torch.cuda.synchronize()
    return dict(out=out, lse=lse, dq=grads[0], dk=grads[1], dv=grads[2], dgate=dgate,
                dbias=dbias)


def _same_bits(a, b):
    return torch.equal(a.view(torch.int16) if a.element_size() == 2 else a.view(torch.int32),
                       b.view(torch.int16) if b.element_size() == 2 else b.view(torch.int32))


@pytest.mark.gpu
@pytest.mark.parametrize("variant_name,world", [("starting", 2), ("starting", 3), ("ending", 2)])
def test_shards_match_whole_problem(variant_name, world):
    import oracle
    from helpers import BF16_REL, assert_close, np64, to_device
    from tri_inputs import ENDING, STARTING, full_mask, make_inputs

    variant = STARTING if variant_name == "starting" else ENDING
    d = make_inputs(264, H=3, c=32, dtype="bf16", seed=41, bias_std=1.4)
    d["mask"] = full_mask(264, seed=41, keep_prob=0.8, fully_masked_rows=(9,))
    g = to_device(d, "cuda:0")
    out, lse = ta.fwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], variant)
    whole = dict(zip(("dq", "dk", "dv", "dbias", "dgate"),
                     ta.bwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], out, lse,
                            g["dout"], variant)))
    whole.update(out=out, lse=lse)
    sh = _run_shards(g, variant, world)
    # every row computed by exactly one shard, with the whole call's bits
    for name in ("out", "lse", "dq", "dk", "dv", "dgate"):
        assert _same_bits(sh[name], whole[name]), name
    # dbias: the same sums in another grouping, rounded once
    assert_close("dbias vs whole", np64(sh["dbias"]), np64(whole["dbias"]), 2e-3)
    ref_b = oracle.bwd(d["q"], d["k"], d["v"], d["bias"], d["gate"], d["dout"], d["mask"],
                       variant)
    assert_close("dbias vs oracle", np64(sh["dbias"]), ref_b[4], BF16_REL)


@pytest.mark.gpu
def test_n768_four_shards():
    """The headline size split over four ranks (192 rows each)."""
    import oracle
    from helpers import BF16_REL, assert_close, np64, to_device
    from tri_inputs import STARTING, workload_inputs

    d = workload_inputs("n768_bf16")
    g = to_device(d, "cuda:0")
    out, lse = ta.fwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], STARTING)
    whole = ta.bwd(g["q"], g["k"], g["v"], g["bias"], g["gate"], g["mask"], out, lse, g["dout"],
                   STARTING)
    sh = _run_shards(g, STARTING, 4)
    assert _same_bits(sh["out"], out) and _same_bits(sh["lse"], lse)
    for name, ref in zip(("dq", "dk", "dv", "dgate"), (whole[0], whole[1], whole[2], whole[4])):
        assert _same_bits(sh[name], ref), name
    assert_close("dbias vs whole", np64(sh["dbias"]), np64(whole[3]), 2e-3)
    rng = np.random.default_rng(7)
    ent = np.stack([rng.integers(0, 4, 32), rng.integers(0, 768, 32), rng.integers(0, 768, 32)],
                   axis=1)
    ref_db = oracle.dbias_entries(d["q"], d["k"], d["v"], d["bias"], d["gate"], d["dout"], ent,
                                  d["mask"], STARTING)
    db = np64(sh["dbias"])[ent[:, 0], ent[:, 1], ent[:, 2]]
    assert_close("dbias (sampled) vs oracle", db, ref_db, BF16_REL)
