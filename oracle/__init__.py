"""fp64 CPU oracle for gated triangle self-attention (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It shares no code with the CUDA library
and never imports it. The arithmetic lives in ``tri_attn_oracle.c`` (plain C,
fp64, libm); this file only builds it and marshals numpy/torch arrays.

Every function takes the inputs exactly as the GPU path receives them (fp32 or
bf16 values, widened to float32 without change) and returns fp64 numpy arrays.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tri_attn_oracle.c")
_LIB = os.path.join(_HERE, "libtri_oracle.so")
_lib = None

STARTING = 0
ENDING = 1


def build(force: bool = False, src: str = _SRC, lib: str = _LIB) -> str:
    """Compile the oracle with gcc (fp64, no fast-math, no FMA contraction, OpenMP)."""
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp, "-lm"])
        os.replace(tmp, lib)
    return lib


def load_library(path: str):
    """Open an oracle shared library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    i32 = ctypes.c_int
    lib.tri_oracle_fwd.argtypes = [i64, i32, i32, i32, P, P, P, P, P, P, i64, P, i64, P, P]
    lib.tri_oracle_probs.argtypes = [i64, i32, i32, i32, P, P, P, P, P, i64, i64, i32, P]
    lib.tri_oracle_bwd.argtypes = [i64, i32, i32, i32, P, P, P, P, P, P, i64, P, P, i64,
                                   P, P, P, P, P]
    lib.tri_oracle_dbias_entries.argtypes = [i64, i32, i32, i32, P, P, P, P, P, P, i64, P,
                                             P, i64, P]
    for f in (lib.tri_oracle_fwd, lib.tri_oracle_probs, lib.tri_oracle_bwd,
              lib.tri_oracle_dbias_entries):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def _f32(x) -> np.ndarray:
    """Widen a torch tensor or numpy array to a contiguous float32 numpy array."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float32).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _u8(m) -> Optional[np.ndarray]:
    if m is None:
        return None
    if hasattr(m, "detach"):
        m = m.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(m, dtype=np.uint8))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _mask_stride(mask: Optional[np.ndarray], N: int) -> int:
    if mask is None:
        return 0
    if mask.ndim == 1:
        assert mask.shape[0] == N
        return 0
    assert mask.shape == (N, N)
    return N


def _dims(q) -> tuple:
    N, N2, H, C = q.shape
    assert N == N2
    return N, H, C


def _rows(rows, N) -> np.ndarray:
    if rows is None:
        rows = np.arange(N, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    assert rows.ndim == 1 and (rows.size == 0 or (rows.min() >= 0 and rows.max() < N))
    return rows


def fwd(q, k, v, bias, gate, mask=None, variant: int = STARTING,
        rows: Optional[Sequence[int]] = None, lib=None):
    """out[n, x, h, c] and lse[n, h, x] for the listed attention rows (all rows
    when rows is None), in the variant's frame."""
    q, k, v, bias, gate = map(_f32, (q, k, v, bias, gate))
    mask = _u8(mask)
    N, H, C = _dims(q)
    rows = _rows(rows, N)
    out = np.zeros((rows.size, N, H, C), dtype=np.float64)
    lse = np.zeros((rows.size, H, N), dtype=np.float64)
    rc = (lib or _load()).tri_oracle_fwd(N, H, C, variant, _ptr(q), _ptr(k), _ptr(v), _ptr(bias),
                                _ptr(gate), _ptr(mask), _mask_stride(mask, N), _ptr(rows),
                                rows.size, _ptr(out), _ptr(lse))
    if rc != 0:
        raise RuntimeError(f"tri_oracle_fwd failed with {rc}")
    return out, lse


def probs(q, k, v, bias, mask=None, variant: int = STARTING, row: int = 0, head: int = 0,
          lib=None):
    """Probability matrix p[x, y] of one attention row and head."""
    q, k, v, bias = map(_f32, (q, k, v, bias))
    mask = _u8(mask)
    N, H, C = _dims(q)
    P = np.zeros((N, N), dtype=np.float64)
    rc = (lib or _load()).tri_oracle_probs(N, H, C, variant, _ptr(q), _ptr(k), _ptr(v), _ptr(bias),
                                  _ptr(mask), _mask_stride(mask, N), row, head, _ptr(P))
    if rc != 0:
        raise RuntimeError(f"tri_oracle_probs failed with {rc}")
    return P


def bwd(q, k, v, bias, gate, dout, mask=None, variant: int = STARTING,
        rows: Optional[Sequence[int]] = None, lib=None):
    """dq, dk, dv, dgate [n, x, h, c] (variant frame) for the listed rows, and
    dbias [H, N, N] (storage layout) summed over the listed rows."""
    q, k, v, bias, gate, dout = map(_f32, (q, k, v, bias, gate, dout))
    mask = _u8(mask)
    N, H, C = _dims(q)
    rows = _rows(rows, N)
    shp = (rows.size, N, H, C)
    dq, dk, dv, dg = (np.zeros(shp, dtype=np.float64) for _ in range(4))
    db = np.zeros((H, N, N), dtype=np.float64)
    rc = (lib or _load()).tri_oracle_bwd(N, H, C, variant, _ptr(q), _ptr(k), _ptr(v), _ptr(bias),
                                _ptr(gate), _ptr(mask), _mask_stride(mask, N), _ptr(dout),
                                _ptr(rows), rows.size, _ptr(dq), _ptr(dk), _ptr(dv),
                                _ptr(dg), _ptr(db))
    if rc != 0:
        raise RuntimeError(f"tri_oracle_bwd failed with {rc}")
    return dq, dk, dv, dg, db


def dbias_entries(q, k, v, bias, gate, dout, entries, mask=None, variant: int = STARTING,
                  lib=None):
    """dbias[h, a, b] (storage layout, summed over all rows) for each (h, a, b)."""
    q, k, v, bias, gate, dout = map(_f32, (q, k, v, bias, gate, dout))
    mask = _u8(mask)
    N, H, C = _dims(q)
    ent = np.ascontiguousarray(np.asarray(entries, dtype=np.int64).reshape(-1, 3))
    out = np.zeros(ent.shape[0], dtype=np.float64)
    rc = (lib or _load()).tri_oracle_dbias_entries(N, H, C, variant, _ptr(q), _ptr(k), _ptr(v),
                                          _ptr(bias), _ptr(gate), _ptr(mask),
                                          _mask_stride(mask, N), _ptr(dout), _ptr(ent),
                                          ent.shape[0], _ptr(out))
    if rc != 0:
        raise RuntimeError(f"tri_oracle_dbias_entries failed with {rc}")
    return out


# ------------------------------------------------ triangle multiplication --

OUTGOING = 0
INCOMING = 1
_MUL_SRC = os.path.join(_HERE, "tri_mul_oracle.c")
_MUL_LIB = os.path.join(_HERE, "libtri_mul_oracle.so")
_mul_lib = None


def load_mul_library(path: str):
    """Open a triangle-multiplication oracle library and declare its signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.tri_mul_oracle_fwd.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, P, P]
    lib.tri_mul_oracle_bwd.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, P, P, P,
                                       P]
    lib.tri_mul_oracle_fwd.restype = ctypes.c_int
    lib.tri_mul_oracle_bwd.restype = ctypes.c_int
    return lib


def build_mul(force: bool = False) -> str:
    return build(force, _MUL_SRC, _MUL_LIB)


def _load_mul():
    global _mul_lib
    if _mul_lib is None:
        _mul_lib = load_mul_library(build_mul())
    return _mul_lib


def _mul_dims(a) -> tuple:
    C, N, N2 = a.shape
    assert N == N2
    return N, C


def mul_fwd(a, b, direction: int = OUTGOING, lib=None) -> np.ndarray:
    """t[c, i, j] of the triangle multiplicative update, channel-major."""
    a, b = map(_f32, (a, b))
    N, C = _mul_dims(a)
    t = np.zeros((C, N, N), dtype=np.float64)
    rc = (lib or _load_mul()).tri_mul_oracle_fwd(N, C, direction, _ptr(a), _ptr(b), _ptr(t))
    if rc != 0:
        raise RuntimeError(f"tri_mul_oracle_fwd failed with {rc}")
    return t


def mul_bwd(a, b, dt, direction: int = OUTGOING, lib=None) -> tuple:
    """(da, db) of L = sum(dt * t), channel-major."""
    a, b, dt = map(_f32, (a, b, dt))
    N, C = _mul_dims(a)
    da = np.zeros((C, N, N), dtype=np.float64)
    db = np.zeros((C, N, N), dtype=np.float64)
    rc = (lib or _load_mul()).tri_mul_oracle_bwd(N, C, direction, _ptr(a), _ptr(b), _ptr(dt),
                                                 _ptr(da), _ptr(db))
    if rc != 0:
        raise RuntimeError(f"tri_mul_oracle_bwd failed with {rc}")
    return da, db


def to_storage(x_rows: np.ndarray, variant: int) -> np.ndarray:
    """Map a full-row result [N(row), N(query), H, C] from the variant frame to
    the storage layout of the pair tensors (a transpose for the ending node)."""
    return x_rows if variant == STARTING else np.ascontiguousarray(x_rows.transpose(1, 0, 2, 3))


from .proj_oracle import (layer_norm, layer_norm_bwd, proj_in_bwd, proj_in_fwd,  # noqa: E402
                          proj_out_bwd, proj_out_fwd)
