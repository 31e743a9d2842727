"""The seeded input recipe (tri_inputs) produces what the design notes state:
shapes, dtypes, distributions, mask counts and determinism per seed. CPU only."""

import numpy as np
import torch

import tri_inputs as ti


def test_workload_shapes_and_masks():
    for name, w in ti.WORKLOADS.items():
        if w.N > 384:
            continue                       # large draws: covered by the GPU tests
        d = ti.workload_inputs(name)
        dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
        for k in ("q", "k", "v", "gate"):
            assert d[k].shape == (w.N, w.N, w.H, w.c) and d[k].dtype == dt
        assert d["bias"].shape == (w.H, w.N, w.N)
        if w.mask == "none":
            assert d["mask"] is None
        else:
            kind, _, n = w.mask.partition(":")
            m = d["mask"].numpy()
            assert m.shape == (w.N,) and int((m == 0).sum()) == int(n)
            if kind == "trailing":
                assert m[w.N - int(n):].sum() == 0 and m[:w.N - int(n)].all()


def test_same_seed_same_draws_and_bias_std():
    a = ti.make_inputs(64, seed=3, bias_std=2.0)
    b = ti.make_inputs(64, seed=3, bias_std=2.0)
    c = ti.make_inputs(64, seed=4, bias_std=2.0)
    assert all(torch.equal(a[k], b[k]) for k in ("q", "k", "v", "gate", "bias", "dout"))
    assert not torch.equal(a["q"], c["q"])
    assert abs(float(a["bias"].float().std()) - 2.0) < 0.05
    assert abs(float(a["q"].float().std()) - 1.0) < 0.02


def test_block_inputs_recipe():
    N, cz, H, c = 16, 128, 4, 32
    d = ti.make_block_inputs(N, cz, H, c, batch=2, seed=5)
    assert d["z"].shape == (2, N, N, cz) and d["z"].dtype == torch.bfloat16
    assert d["w_qkvg"].shape == (cz, 4 * H * c) and d["w_b"].shape == (cz, H)
    assert d["w_o"].shape == (H * c, cz) and d["dbias"].shape == (2, H, N, N)
    for k in ("gamma", "beta", "b_g", "b_o"):
        assert d[k].dtype == torch.float32
    z = d["z"].float().numpy()
    # a per-row offset on top of N(0, 1): the row means spread like N(0, 1)
    assert 0.8 < float(np.std(z.mean(axis=-1))) < 1.2
    assert 0.9 < float(np.mean(z.std(axis=-1))) < 1.1
    assert abs(float(d["gamma"].mean()) - 1.0) < 0.03
    assert abs(float(d["w_qkvg"].float().std()) - cz ** -0.5) < 0.005
    assert abs(float(d["w_o"].float().std()) - (H * c) ** -0.5) < 0.005
    again = ti.make_block_inputs(N, cz, H, c, batch=2, seed=5)
    assert all(torch.equal(d[k], again[k]) for k in d if k != "meta")
