"""Seeded synthetic inputs for gated triangle self-attention.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic. Both the CUDA path and the fp64 oracle receive exactly the
tensors produced here.

Recipe (one rule for every workload):
  * generator: ``numpy.random.default_rng(seed)`` (PCG64);
  * draw order: q, k, v, gate, bias, dout, then the mask choice;
  * values: ``standard_normal(dtype=float32) * std``, then rounded to the
    storage dtype (bf16 by round-to-nearest-even through torch);
  * pair tensors q, k, v, gate, dout are [N, N, H, c] (c fastest); bias is
    [H, N, N]; the key mask is uint8 [N] (1 = key takes part), shared by every
    attention row (row stride 0), or None for "all ones".

The workloads mirror the crop sizes the pages name for AlphaFold-family
training (TurboPairFormer news page, "Benchmark di addestramento": crops
384/640/768) plus a small fp32 case and a long-sequence inference case.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

STARTING = 0
ENDING = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    H: int = 4
    c: int = 32
    dtype: str = "bf16"          # "f32" or "bf16"
    variants: tuple = (STARTING,)
    bias_std: float = 1.0
    mask: str = "none"           # "none" | "random:<count>" | "trailing:<count>"
    backward: bool = True
    seed: int = 0


# The five workloads: sizes, distributions and masks of the scope statement.
WORKLOADS = {
    "n32_f32": Workload("n32_f32", N=32, dtype="f32"),
    # 10% of 256 keys = 25.6 -> 26 keys, drawn without replacement.
    "n256_bf16": Workload("n256_bf16", N=256, bias_std=float(np.sqrt(2.0)),
                          mask="random:26"),
    "n384_bf16": Workload("n384_bf16", N=384, bias_std=float(np.sqrt(2.0)),
                          mask="trailing:32", variants=(STARTING, ENDING)),
    "n768_bf16": Workload("n768_bf16", N=768),
    # 5% of 1536 = 76.8 -> 77 trailing keys.
    "n1536_bf16_fwd": Workload("n1536_bf16_fwd", N=1536, mask="trailing:77",
                               backward=False),
}


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(x)
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t.to(torch.float32)
    raise ValueError(f"unknown dtype {dtype!r}")


def make_mask(rng: np.random.Generator, N: int, spec: str) -> Optional[torch.Tensor]:
    """Key mask of shape [N] (uint8, 1 = key takes part) or None for all ones."""
    if spec == "none":
        return None
    kind, _, count = spec.partition(":")
    n = int(count)
    m = np.ones(N, dtype=np.uint8)
    if kind == "random":
        m[rng.choice(N, size=n, replace=False)] = 0
    elif kind == "trailing":
        if n > 0:
            m[N - n:] = 0
    else:
        raise ValueError(f"unknown mask spec {spec!r}")
    return torch.from_numpy(m)


def make_inputs(N: int, H: int = 4, c: int = 32, dtype: str = "bf16", seed: int = 0,
                bias_std: float = 1.0, mask: str = "none", backward: bool = True,
                std: float = 1.0) -> dict:
    """Draw one problem. Returns CPU tensors q, k, v, gate, bias, dout (None when
    backward is False) and mask (None or uint8 [N])."""
    rng = np.random.default_rng(seed)
    pair = (N, N, H, c)

    def draw(shape, s):
        return _round(rng.standard_normal(shape, dtype=np.float32) * np.float32(s), dtype)

    out = {}
    out["q"] = draw(pair, std)
    out["k"] = draw(pair, std)
    out["v"] = draw(pair, std)
    out["gate"] = draw(pair, std)
    out["bias"] = draw((H, N, N), bias_std)
    out["dout"] = draw(pair, std) if backward else None
    out["mask"] = make_mask(rng, N, mask)
    out["meta"] = dict(N=N, H=H, c=c, dtype=dtype, seed=seed, bias_std=bias_std,
                       mask=mask)
    return out


def workload_inputs(name: str, seed: Optional[int] = None) -> dict:
    w = WORKLOADS[name]
    return make_inputs(w.N, w.H, w.c, w.dtype, w.seed if seed is None else seed,
                       bias_std=w.bias_std, mask=w.mask, backward=w.backward)


def full_mask(N: int, seed: int, keep_prob: float = 0.8, fully_masked_rows=()) -> torch.Tensor:
    """A per-row key mask [N, N] (row stride N) for edge-case tests: each entry is
    kept with probability keep_prob; rows listed in fully_masked_rows mask every key."""
    rng = np.random.default_rng(seed + 7919)
    m = (rng.random((N, N)) < keep_prob).astype(np.uint8)
    for r in fully_masked_rows:
        m[r, :] = 0
    return torch.from_numpy(m)


def make_block_inputs(N: int, cz: int = 128, H: int = 4, c: int = 32, batch: Optional[int] = None,
                      seed: int = 0) -> dict:
    """Draw the pair representation, the parameters of the block around the
    attention (LayerNorm and projections) and the gradients that flow into it.

    Draw order: z, gamma, beta, w_qkvg, b_g, w_b, w_o, b_o, then the incoming
    gradients dq, dk, dv, dg, dbias (same shapes as q, k, v, g, bias) and dy.
    z ~ N(0, 1) + a per-row offset N(0, 1) (LayerNorm must remove it); gamma ~
    1 + 0.1 N(0, 1); beta, b_g, b_o ~ 0.1 N(0, 1); weights ~ N(0, 1/fan_in);
    gradients ~ N(0, 1). Activations and weights are bf16, the LayerNorm
    parameters and biases float32. With batch=None the pair tensors are
    [N, N, ...], else [batch, N, N, ...]."""
    rng = np.random.default_rng(seed)
    lead = (N, N) if batch is None else (batch, N, N)
    hc = H * c

    def draw(shape, s=1.0, shift=0.0, dtype="bf16"):
        x = rng.standard_normal(shape, dtype=np.float32) * np.float32(s) + np.float32(shift)
        return _round(x, dtype)

    z = rng.standard_normal(lead + (cz,), dtype=np.float32)
    z += rng.standard_normal(lead + (1,), dtype=np.float32)
    out = {"z": _round(z, "bf16"),
           "gamma": draw((cz,), 0.1, 1.0, "f32"), "beta": draw((cz,), 0.1, 0.0, "f32"),
           "w_qkvg": draw((cz, 4 * hc), cz ** -0.5), "b_g": draw((hc,), 0.1, 0.0, "f32"),
           "w_b": draw((cz, H), cz ** -0.5), "w_o": draw((hc, cz), hc ** -0.5),
           "b_o": draw((cz,), 0.1, 0.0, "f32")}
    for name in ("dq", "dk", "dv", "dg"):
        out[name] = draw(lead + (H, c))
    out["dbias"] = draw(lead[:-2] + (H, N, N))
    out["dy"] = draw(lead + (cz,))
    out["meta"] = dict(N=N, cz=cz, H=H, c=c, batch=batch, seed=seed)
    return out


def make_update_inputs(N: int, cz: int = 128, c: int = 128, seed: int = 0) -> dict:
    """Draw the pair representation, the parameters of the triangle
    multiplicative update and the gradient that flows into its output.

    Draw order: z, ln_gamma, ln_beta, w_in, b_in, ln_out_gamma, ln_out_beta, w_o,
    b_o, dy. z ~ N(0, 1) + a per-position offset N(0, 1); LayerNorm gains ~
    1 + 0.1 N(0, 1); offsets and biases ~ 0.1 N(0, 1); w_in ~ N(0, 1/cz) (its
    [cz][4c + cz] columns are W_ap, W_ag, W_bp, W_bg, W_g); w_o ~ N(0, 1/c); dy ~
    N(0, 1). z, w_in, w_o and dy are bf16, the rest float32."""
    rng = np.random.default_rng(seed)

    def draw(shape, s=1.0, shift=0.0, dtype="bf16"):
        x = rng.standard_normal(shape, dtype=np.float32) * np.float32(s) + np.float32(shift)
        return _round(x, dtype)

    z = rng.standard_normal((N, N, cz), dtype=np.float32)
    z += rng.standard_normal((N, N, 1), dtype=np.float32)
    p = {"ln_gamma": draw((cz,), 0.1, 1.0, "f32"), "ln_beta": draw((cz,), 0.1, 0.0, "f32"),
         "w_in": draw((cz, 4 * c + cz), cz ** -0.5), "b_in": draw((4 * c + cz,), 0.1, 0.0, "f32"),
         "ln_out_gamma": draw((c,), 0.1, 1.0, "f32"), "ln_out_beta": draw((c,), 0.1, 0.0, "f32"),
         "w_o": draw((c, cz), c ** -0.5), "b_o": draw((cz,), 0.1, 0.0, "f32")}
    dy = draw((N, N, cz))
    return {"z": _round(z, "bf16"), "params": p, "dy": dy,
            "meta": dict(N=N, cz=cz, c=c, seed=seed)}
