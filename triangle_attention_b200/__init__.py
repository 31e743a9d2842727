"""Thin Python binding of libtri_attn.so (gated triangle self-attention, B200).

Argument marshalling only: every step of the computation runs in the CUDA
library. PyTorch supplies device memory and the current stream. If the shared
library is missing or cannot be loaded, every entry point raises; there is no
CPU fallback.

Entry points (names follow the C ABI in include/tri_attn.h):
    fwd(q, k, v, bias, gate, mask=None, variant=STARTING) -> (out, lse)
    bwd(q, k, v, bias, gate, mask, out, lse, dout, variant) -> (dq, dk, dv, dbias, dgate)
    fwd_workspace_size / bwd_workspace_size / read_status
    TriangleAttention: torch.autograd.Function over fwd/bwd.
    mul_fwd / mul_bwd, TriangleMultiplication: the triangle multiplicative update.
    proj_in_fwd / proj_in_bwd / proj_out_fwd / proj_out_bwd: LayerNorm and the
    projections around the attention; TriangleAttentionBlock chains them.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

STARTING = 0
ENDING = 1
F32 = 0
BF16 = 1

STATUS = {
    0: "ok", 1: "invalid argument", 2: "unsupported problem", 3: "workspace missing or too small",
    4: "CUDA call failed", 5: "device wait timed out", 6: "device index check failed",
}

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtri_attn.so")
_lib = None


class TriAttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, 'unknown status')} ({code})")
        self.code = code


class LaunchOpts(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("flags", ctypes.c_uint32),
                ("main_start", ctypes.c_void_p), ("main_stop", ctypes.c_void_p),
                ("out_residual", ctypes.c_void_p)]


OPT_ONCHIP_SUMS = 0x1
OPT_EXP2_SPLIT = 0x2


def launch_opts(main_start=None, main_stop=None, residual=None,
                onchip_sums: bool = False, exp2_split: bool = False) -> LaunchOpts:
    """Options: torch.cuda.Event objects recorded around the main kernel, the
    bf16 rounding residual of `out` (a tensor shaped like out) that the
    forward writes and the backward uses for D and dgate, (backward only) the
    on-chip summation of the tile contributions (TRI_ATTN_OPT_ONCHIP_SUMS) and
    (forward only) one exponential pair in four on the FMA pipe
    (TRI_ATTN_OPT_EXP2_SPLIT)."""
    def handle(ev):
        if ev is None:
            return None
        if not ev.cuda_event:            # torch creates the event lazily
            ev.record()
        return ctypes.c_void_p(ev.cuda_event)
    flags = (OPT_ONCHIP_SUMS if onchip_sums else 0) | (OPT_EXP2_SPLIT if exp2_split else 0)
    return LaunchOpts(ctypes.sizeof(LaunchOpts), flags,
                      handle(main_start), handle(main_stop),
                      None if residual is None else ctypes.c_void_p(residual.data_ptr()))


def _with_residual(opts, residual):
    if residual is None:
        return opts
    if opts is None:
        return launch_opts(residual=residual)
    opts.out_residual = ctypes.c_void_p(residual.data_ptr())
    return opts


OUTGOING, INCOMING = 0, 1


class MulProblem(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("C", ctypes.c_int32), ("direction", ctypes.c_int32)]


class MulUpdateProblem(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("cz", ctypes.c_int32), ("c", ctypes.c_int32),
                ("direction", ctypes.c_int32), ("eps", ctypes.c_float)]


MUL_UPDATE_PARAMS = ("ln_gamma", "ln_beta", "w_in", "b_in", "ln_out_gamma", "ln_out_beta",
                     "w_o", "b_o")


class MulUpdateParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in MUL_UPDATE_PARAMS]


class MulUpdateGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in MUL_UPDATE_PARAMS]


class ProjProblem(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("batch", ctypes.c_int32), ("cz", ctypes.c_int32),
                ("H", ctypes.c_int32), ("c", ctypes.c_int32), ("eps", ctypes.c_float),
                ("reserved", ctypes.c_int32)]


class Problem(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("H", ctypes.c_int32), ("c", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("variant", ctypes.c_int32),
                ("mask_row_stride", ctypes.c_int64), ("batch", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


def lib():
    """The loaded library; raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m triangle_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        PP = ctypes.POINTER(Problem)
        sz = ctypes.c_size_t
        L.tri_attn_version.restype = ctypes.c_int
        L.tri_attn_status_string.argtypes = [ctypes.c_int]
        L.tri_attn_status_string.restype = ctypes.c_char_p
        L.tri_attn_last_cuda_error.argtypes = []
        L.tri_attn_last_cuda_error.restype = ctypes.c_char_p
        L.tri_attn_fwd_workspace_size.argtypes = [PP, ctypes.POINTER(sz)]
        L.tri_attn_bwd_workspace_size.argtypes = [PP, ctypes.POINTER(sz)]
        PO = ctypes.POINTER(LaunchOpts)
        L.tri_attn_fwd.argtypes = [PP, P, P, P, P, P, P, P, P, P, sz, P]
        L.tri_attn_bwd.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, sz, P]
        L.tri_attn_fwd_ex.argtypes = [PP, P, P, P, P, P, P, P, P, P, sz, P, PO]
        L.tri_attn_bwd_ex.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, sz, P, PO]
        L.tri_attn_kernel_launches.argtypes = [PP, ctypes.c_int, ctypes.c_int,
                                               ctypes.POINTER(ctypes.c_int32)]
        L.tri_attn_read_status.argtypes = [P, ctypes.POINTER(ctypes.c_int32), P]
        L.tri_attn_get_status.argtypes = [P, P]
        L.tri_attn_check_exp2.argtypes = [P, P, P, ctypes.c_int64, P]
        L.tri_attn_probe_mma.argtypes = [ctypes.c_int32] * 4 + [P, P, P]
        i64 = ctypes.c_int64
        L.tri_attn_fwd_rows.argtypes = [PP, i64, i64, P, P, P, P, P, P, P, P, P, sz, P]
        L.tri_attn_bwd_rows.argtypes = [PP, i64, i64] + [P] * 15 + [sz, P]
        L.tri_attn_dbias_reduce.argtypes = [P, ctypes.c_int32, i64, ctypes.c_int32, P, P]
        L.tri_attn_check_wait_timeout.argtypes = [P, sz, P]
        MP = ctypes.POINTER(MulProblem)
        L.tri_mul_workspace_size.argtypes = [MP, ctypes.POINTER(sz)]
        L.tri_mul_fwd.argtypes = [MP, P, P, P, P, sz, P]
        L.tri_mul_bwd.argtypes = [MP, P, P, P, P, P, P, sz, P]
        UP = ctypes.POINTER(MulUpdateProblem)
        L.tri_mul_update_sizes.argtypes = [UP, ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.tri_mul_update_fwd.argtypes = [UP, ctypes.POINTER(MulUpdateParams), P, P, P, sz, P,
                                         sz, P]
        L.tri_mul_update_bwd.argtypes = [UP, ctypes.POINTER(MulUpdateParams), P, P, sz, P, P,
                                         ctypes.POINTER(MulUpdateGrads), P, sz, P]
        JP = ctypes.POINTER(ProjProblem)
        L.tri_proj_workspace_size.argtypes = [JP, ctypes.POINTER(sz)]
        L.tri_proj_in_fwd.argtypes = [JP] + [P] * 13 + [P, sz, P]
        L.tri_proj_in_bwd.argtypes = [JP] + [P] * 17 + [P, sz, P]
        L.tri_proj_out_fwd.argtypes = [JP] + [P] * 4 + [P, sz, P]
        L.tri_proj_out_bwd.argtypes = [JP] + [P] * 6 + [P, sz, P]
        for f in (L.tri_attn_fwd_workspace_size, L.tri_attn_bwd_workspace_size, L.tri_attn_fwd,
                  L.tri_attn_bwd, L.tri_attn_fwd_ex, L.tri_attn_bwd_ex,
                  L.tri_attn_kernel_launches, L.tri_attn_read_status, L.tri_attn_get_status,
                  L.tri_attn_fwd_rows, L.tri_attn_bwd_rows, L.tri_attn_dbias_reduce,
                  L.tri_attn_check_exp2, L.tri_attn_probe_mma,
                  L.tri_attn_check_wait_timeout, L.tri_mul_workspace_size, L.tri_mul_fwd,
                  L.tri_mul_bwd, L.tri_mul_update_sizes, L.tri_mul_update_fwd,
                  L.tri_mul_update_bwd, L.tri_proj_workspace_size, L.tri_proj_in_fwd,
                  L.tri_proj_in_bwd, L.tri_proj_out_fwd, L.tri_proj_out_bwd):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def problem(q: torch.Tensor, mask: Optional[torch.Tensor], variant: int) -> Problem:
    """The problem of pair tensors [N, N, H, c], or of a batch [B, N, N, H, c]
    (mask None, [N] or [N, N] unbatched; None, [B, N] or [B, N, N] batched)."""
    if q.dim() not in (4, 5) or q.shape[-4] != q.shape[-3]:
        raise ValueError(f"pair tensors must be [N, N, H, c] or [B, N, N, H, c], "
                         f"got {tuple(q.shape)}")
    N, _, H, c = q.shape[-4:]
    B = q.shape[0] if q.dim() == 5 else 1
    lead = q.dim() - 4
    stride = 0
    if mask is not None:
        if mask.dim() - lead == 1 and mask.shape[-1] == N:
            stride = 0
        elif mask.dim() - lead == 2 and tuple(mask.shape[-2:]) == (N, N):
            stride = N
        else:
            raise ValueError("mask must be [N] (shared by every row) or [N, N], with the "
                             "pair tensors' leading batch dimension if they have one")
        if lead and mask.shape[0] != B:
            raise ValueError(f"mask batch {mask.shape[0]} != {B}")
    return Problem(N, H, c, _dtype_code(q), variant, stride, B, 0)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(code: int, where: str):
    if code != 0:
        if code == 4:   # TRI_ATTN_ERR_CUDA: name the CUDA error behind it
            where = f"{where} [{lib().tri_attn_last_cuda_error().decode()}]"
        raise TriAttnError(code, where)


def fwd_workspace_size(prob: Problem) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().tri_attn_fwd_workspace_size(ctypes.byref(prob), ctypes.byref(n)),
           "tri_attn_fwd_workspace_size")
    return n.value


def bwd_workspace_size(prob: Problem) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().tri_attn_bwd_workspace_size(ctypes.byref(prob), ctypes.byref(n)),
           "tri_attn_bwd_workspace_size")
    return n.value


def kernel_launches(prob: Problem, backward: bool, has_mask: bool,
                    onchip_sums: bool = False) -> int:
    """Kernel launches one forward (backward=False) or backward call enqueues
    (onchip_sums: the backward with OPT_ONCHIP_SUMS)."""
    n = ctypes.c_int32(0)
    code = (2 if onchip_sums else 1) if backward else 0
    _check(lib().tri_attn_kernel_launches(ctypes.byref(prob), code, int(has_mask),
                                          ctypes.byref(n)), "tri_attn_kernel_launches")
    return n.value


def workspace(nbytes: int, device) -> torch.Tensor:
    """A device buffer for the library's scratch (torch allocations are
    256-byte aligned)."""
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("every tensor must be contiguous")


def fwd(q, k, v, bias, gate, mask=None, variant: int = STARTING, out=None, lse=None, ws=None,
        stream=None, opts: Optional[LaunchOpts] = None, residual=None):
    """Forward. Returns (out, lse); out has q's dtype, lse is float32 [N, H, N]
    ([B, N, H, N] for a batch [B, N, N, H, c], whose B problems share each
    launch). residual (bf16 path): a tensor shaped like out that receives
    out's rounding residual, for the compensated backward."""
    _contig(q, k, v, bias, gate, mask, residual)
    opts = _with_residual(opts, residual)
    prob = problem(q, mask, variant)
    N, _, H, _ = q.shape[-4:]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:-4] + (N, H, N), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(fwd_workspace_size(prob), q.device)
    _check(lib().tri_attn_fwd_ex(ctypes.byref(prob), _p(q), _p(k), _p(v), _p(bias), _p(gate),
                                 _p(mask), _p(out), _p(lse), _p(ws), ws.numel(), _stream(stream),
                                 None if opts is None else ctypes.byref(opts)),
           "tri_attn_fwd")
    return out, lse


def bwd(q, k, v, bias, gate, mask, out, lse, dout, variant: int = STARTING, grads=None, ws=None,
        stream=None, opts: Optional[LaunchOpts] = None, residual=None):
    """Backward. Returns (dq, dk, dv, dbias, dgate) in the inputs' dtype.
    residual: the tensor the forward filled, to form D and dgate from out plus
    its rounding residual."""
    _contig(q, k, v, bias, gate, mask, out, lse, dout, residual)
    opts = _with_residual(opts, residual)
    prob = problem(q, mask, variant)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                 torch.empty_like(bias), torch.empty_like(gate))
    dq, dk, dv, dbias, dgate = grads
    if ws is None:
        ws = workspace(bwd_workspace_size(prob), q.device)
    _check(lib().tri_attn_bwd_ex(ctypes.byref(prob), _p(q), _p(k), _p(v), _p(bias), _p(gate),
                                 _p(mask), _p(out), _p(lse), _p(dout), _p(dq), _p(dk), _p(dv),
                                 _p(dbias), _p(dgate), _p(ws), ws.numel(), _stream(stream),
                                 None if opts is None else ctypes.byref(opts)),
           "tri_attn_bwd")
    return dq, dk, dv, dbias, dgate


# ------------------------------------------------------------ row shards --

def shard_rows(N: int, world: int, rank: int) -> tuple:
    """(row_begin, row_count) of rank `rank` when the N attention rows are split
    into `world` contiguous shards of whole 8-row groups; the first
    (N/8) mod world ranks take one group more."""
    if world < 1 or not 0 <= rank < world or N % 8:
        raise ValueError(f"cannot shard N={N} rows over {world} ranks (rank {rank})")
    base, extra = divmod(N // 8, world)
    begin = 8 * (rank * base + min(rank, extra))
    return begin, 8 * (base + (1 if rank < extra else 0))


def fwd_rows(q, k, v, bias, gate, mask, variant: int, row_begin: int, row_count: int,
             out=None, lse=None, ws=None, stream=None):
    """Forward of the attention rows [row_begin, row_begin + row_count) (bf16).
    Inputs and outputs are the full tensors; only the shard's rows of out and
    lse are written (the rest of freshly allocated outputs is undefined)."""
    _contig(q, k, v, bias, gate, mask)
    prob = problem(q, mask, variant)
    N, H = q.shape[0], q.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((N, H, N), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(fwd_workspace_size(prob), q.device)
    _check(lib().tri_attn_fwd_rows(ctypes.byref(prob), row_begin, row_count, _p(q), _p(k), _p(v),
                                   _p(bias), _p(gate), _p(mask), _p(out), _p(lse), _p(ws),
                                   ws.numel(), _stream(stream)), "tri_attn_fwd_rows")
    return out, lse


def bwd_rows(q, k, v, bias, gate, mask, out, lse, dout, variant: int, row_begin: int,
             row_count: int, grads=None, ws=None, stream=None):
    """Backward of a row shard. Returns (dq, dk, dv, dbias_partial, dgate): the
    shard's rows of the pair gradients (full tensors, other rows untouched) and
    the fp32 [H, N, N] sum of dbias over the shard's rows."""
    _contig(q, k, v, bias, gate, mask, out, lse, dout)
    prob = problem(q, mask, variant)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                 torch.empty(bias.shape, dtype=torch.float32, device=q.device),
                 torch.empty_like(gate))
    dq, dk, dv, dbp, dgate = grads
    if ws is None:
        ws = workspace(bwd_workspace_size(prob), q.device)
    _check(lib().tri_attn_bwd_rows(ctypes.byref(prob), row_begin, row_count, _p(q), _p(k), _p(v),
                                   _p(bias), _p(gate), _p(mask), _p(out), _p(lse), _p(dout),
                                   _p(dq), _p(dk), _p(dv), _p(dbp), _p(dgate), _p(ws), ws.numel(),
                                   _stream(stream)), "tri_attn_bwd_rows")
    return dq, dk, dv, dbp, dgate


def dbias_reduce(partials: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """bf16 dbias [H, N, N] = the fp32 partials [W, H, N, N] summed over W in
    index order (rank order) and rounded once, on the GPU."""
    _contig(partials)
    W, H, N, _ = partials.shape
    if out is None:
        out = torch.empty((H, N, N), dtype=torch.bfloat16, device=partials.device)
    _check(lib().tri_attn_dbias_reduce(_p(partials), W, N, H, _p(out), _stream(stream)),
           "tri_attn_dbias_reduce")
    return out


def gather_partials(partial: torch.Tensor, group=None) -> torch.Tensor:
    """[W, ...] stack of every rank's `partial`, in rank order (torch.distributed
    all_gather; NCCL on GPUs, any backend's tensors work)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = [torch.empty_like(partial) for _ in range(world)]
    dist.all_gather(parts, partial.contiguous(), group=group)
    return torch.stack(parts)


def sharded_bwd(q, k, v, bias, gate, mask, out, lse, dout, variant: int = STARTING, group=None,
                ws=None, stream=None):
    """Backward of one problem split by rows over the ranks of `group`: each
    rank computes its shard's rows of dq, dk, dv and dgate, the dbias partials
    are all-gathered and summed in rank order on the GPU, so every rank holds
    the same full dbias. Returns (dq, dk, dv, dbias, dgate, (row_begin, row_count))."""
    import torch.distributed as dist
    rows = shard_rows(q.shape[0], dist.get_world_size(group), dist.get_rank(group))
    dq, dk, dv, dbp, dgate = bwd_rows(q, k, v, bias, gate, mask, out, lse, dout, variant,
                                      rows[0], rows[1], ws=ws, stream=stream)
    dbias = dbias_reduce(gather_partials(dbp, group), stream=stream)
    return dq, dk, dv, dbias, dgate, rows


def read_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns the device status word of the last
    call that used this workspace (0 = ok)."""
    v = ctypes.c_int32(0)
    _check(lib().tri_attn_read_status(_p(ws), ctypes.byref(v), _stream(stream)),
           "tri_attn_read_status")
    return v.value


def get_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns the device status word of the last
    call that used this workspace as a status code (0 = ok); raises only if the
    query itself fails."""
    code = lib().tri_attn_get_status(_p(ws), _stream(stream))
    if code == 4:
        _check(code, "tri_attn_get_status")
    return code


def probe_mma(n: int, layout: int = 0, instructions: int = 16384, ctas: int = 148,
              device="cuda") -> float:
    """Mean SM cycles per tcgen05.mma (M=128, K=16, N=n) issued back to back,
    over `ctas` CTAs; raises if a completion wait ran out."""
    cycles = torch.zeros(ctas, dtype=torch.int64, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    _check(lib().tri_attn_probe_mma(n, layout, ctas, instructions, _p(cycles), _p(status),
                                    _stream()), "tri_attn_probe_mma")
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise TriAttnError(int(status.item()), "tri_attn_probe_mma")
    issued = (instructions + 7) // 8 * 8
    return float(cycles.double().mean().item()) / issued


def check_exp2(x: torch.Tensor, stream=None) -> tuple:
    """(FMA-pipe exp2, MUFU exp2) of the fp32 device tensor x, elementwise."""
    _contig(x)
    y_fma, y_mufu = torch.empty_like(x), torch.empty_like(x)
    _check(lib().tri_attn_check_exp2(_p(x), _p(y_fma), _p(y_mufu), x.numel(), _stream(stream)),
           "tri_attn_check_exp2")
    return y_fma, y_mufu


def check_wait_timeout(ws: torch.Tensor, stream=None) -> int:
    """Runs the diagnostic kernel whose bounded wait nothing satisfies and
    returns the status word it leaves (TIMEOUT when the wait gave up)."""
    _check(lib().tri_attn_check_wait_timeout(_p(ws), ws.numel(), _stream(stream)),
           "tri_attn_check_wait_timeout")
    return read_status(ws, stream)


def _mul_problem(a: torch.Tensor, direction: int) -> MulProblem:
    C, N, N2 = a.shape
    if N != N2 or a.dtype != torch.bfloat16:
        raise ValueError("triangle multiplication takes bf16 [C, N, N] stacks")
    return MulProblem(N, C, direction)


def mul_fwd(a, b, direction: int = OUTGOING, t=None, ws=None, stream=None) -> torch.Tensor:
    """Triangle multiplicative update contraction, channel-major bf16 [C, N, N]:
    outgoing t[c,i,j] = sum_k a[c,i,k] b[c,j,k]; incoming sum_k a[c,k,i] b[c,k,j]."""
    _contig(a, b, t)
    prob = _mul_problem(a, direction)
    if t is None:
        t = torch.empty_like(a)
    if ws is None:
        ws = workspace(256, a.device)
    _check(lib().tri_mul_fwd(ctypes.byref(prob), _p(a), _p(b), _p(t), _p(ws), ws.numel(),
                             _stream(stream)), "tri_mul_fwd")
    return t


def mul_bwd(a, b, dt, direction: int = OUTGOING, grads=None, ws=None, stream=None) -> tuple:
    """(da, db) of L = sum(dt * t) for mul_fwd(a, b, direction)."""
    _contig(a, b, dt)
    prob = _mul_problem(a, direction)
    da, db = grads if grads is not None else (torch.empty_like(a), torch.empty_like(b))
    if ws is None:
        ws = workspace(256, a.device)
    _check(lib().tri_mul_bwd(ctypes.byref(prob), _p(a), _p(b), _p(dt), _p(da), _p(db), _p(ws),
                             ws.numel(), _stream(stream)), "tri_mul_bwd")
    return da, db


class TriangleAttention(torch.autograd.Function):
    """out = TriangleAttention.apply(q, k, v, bias, gate, mask, variant).

    Unbatched: q, k, v, gate [N, N, H, c], bias [H, N, N], mask None, [N] or
    [N, N]. Batched: a leading batch dimension on every tensor (q [B, N, N, H,
    c], bias [B, H, N, N], mask None, [B, N] or [B, N, N]); each batch element
    is an independent problem, and the B problems share each kernel launch."""

    @staticmethod
    def forward(ctx, q, k, v, bias, gate, mask=None, variant=STARTING):
        ctx.mask = mask
        ctx.variant = variant
        out, lse = fwd(q, k, v, bias, gate, mask, variant)
        ctx.save_for_backward(q, k, v, bias, gate, out, lse)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, bias, gate, out, lse = ctx.saved_tensors
        dq, dk, dv, dbias, dgate = bwd(q, k, v, bias, gate, ctx.mask, out, lse,
                                       dout.contiguous(), ctx.variant)
        return dq, dk, dv, dbias, dgate, None, None


def triangle_attention(q, k, v, bias, gate, mask=None, variant: int = STARTING) -> torch.Tensor:
    """Gated triangle self-attention with pair bias (differentiable), unbatched or
    with a leading batch dimension; see TriangleAttention."""
    return TriangleAttention.apply(q, k, v, bias, gate, mask, variant)


class TriangleMultiplication(torch.autograd.Function):
    """t = TriangleMultiplication.apply(a, b, direction) on channel-major bf16
    stacks [C, N, N] (or [B, C, N, N], each batch element in turn)."""

    @staticmethod
    def forward(ctx, a, b, direction=OUTGOING):
        ctx.direction = direction
        ctx.save_for_backward(a, b)
        if a.dim() == 3:
            return mul_fwd(a, b, direction)
        t = torch.empty_like(a)
        for i in range(a.shape[0]):
            mul_fwd(a[i], b[i], direction, t=t[i])
        return t

    @staticmethod
    def backward(ctx, dt):
        a, b = ctx.saved_tensors
        dt = dt.contiguous()
        if a.dim() == 3:
            da, db = mul_bwd(a, b, dt, ctx.direction)
        else:
            da, db = torch.empty_like(a), torch.empty_like(b)
            for i in range(a.shape[0]):
                mul_bwd(a[i], b[i], dt[i], ctx.direction, grads=(da[i], db[i]))
        return da, db, None


# --------------------------------------- full triangle multiplicative update --

def _update_problem(z: torch.Tensor, params: dict, direction: int, eps: float):
    if z.dim() != 3 or z.shape[0] != z.shape[1] or z.dtype != torch.bfloat16:
        raise ValueError("the update takes a bf16 pair tensor [N, N, cz]")
    N, cz = z.shape[0], z.shape[2]
    c = (params["w_in"].shape[1] - cz) // 4
    return MulUpdateProblem(N, cz, c, direction, eps)


def _update_params(params: dict) -> MulUpdateParams:
    _contig(*[params[n] for n in MUL_UPDATE_PARAMS])
    return MulUpdateParams(*[params[n].data_ptr() for n in MUL_UPDATE_PARAMS])


def mul_update_sizes(prob: MulUpdateProblem) -> tuple:
    saved, ws = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib().tri_mul_update_sizes(ctypes.byref(prob), ctypes.byref(saved), ctypes.byref(ws)),
           "tri_mul_update_sizes")
    return saved.value, ws.value


def mul_update_fwd(z, params: dict, direction: int = OUTGOING, eps: float = 1e-5, ws=None,
                   stream=None) -> tuple:
    """The full triangle multiplicative update, bf16 [N, N, cz] -> [N, N, cz].
    params: ln_gamma, ln_beta [cz], w_in [cz, 4c + cz] (bf16; W_ap W_ag W_bp W_bg
    W_g), b_in [4c + cz], ln_out_gamma, ln_out_beta [c], w_o [c, cz] (bf16), b_o
    [cz]; float32 unless marked. Returns (y, saved): saved holds the activations
    the backward reads."""
    _contig(z)
    prob = _update_problem(z, params, direction, eps)
    nsaved, nws = mul_update_sizes(prob)
    saved = workspace(nsaved, z.device)
    if ws is None:
        ws = workspace(nws, z.device)
    y = torch.empty_like(z)
    pp = _update_params(params)
    _check(lib().tri_mul_update_fwd(ctypes.byref(prob), ctypes.byref(pp), _p(z), _p(y),
                                    _p(saved), saved.numel(), _p(ws), ws.numel(),
                                    _stream(stream)), "tri_mul_update_fwd")
    return y, saved


def mul_update_bwd(z, params: dict, saved, dy, direction: int = OUTGOING, eps: float = 1e-5,
                   ws=None, stream=None) -> tuple:
    """(dz, grads) of L = sum(dy * y) for mul_update_fwd; grads maps every
    parameter name to its float32 gradient."""
    _contig(z, dy, saved)
    prob = _update_problem(z, params, direction, eps)
    _, nws = mul_update_sizes(prob)
    if ws is None:
        ws = workspace(nws, z.device)
    dz = torch.empty_like(z)
    grads = {n: torch.empty(params[n].shape, dtype=torch.float32, device=z.device)
             for n in MUL_UPDATE_PARAMS}
    gg = MulUpdateGrads(*[grads[n].data_ptr() for n in MUL_UPDATE_PARAMS])
    pp = _update_params(params)
    _check(lib().tri_mul_update_bwd(ctypes.byref(prob), ctypes.byref(pp), _p(z), _p(saved),
                                    saved.numel(), _p(dy), _p(dz), ctypes.byref(gg), _p(ws),
                                    ws.numel(), _stream(stream)), "tri_mul_update_bwd")
    return dz, grads


class TriangleMultiplicativeUpdate(torch.autograd.Function):
    """y = TriangleMultiplicativeUpdate.apply(z, direction, eps, *params) with the
    parameters in MUL_UPDATE_PARAMS order; gradients for z and every parameter
    (cast to each parameter's dtype)."""

    @staticmethod
    def forward(ctx, z, direction, eps, *plist):
        params = dict(zip(MUL_UPDATE_PARAMS, plist))
        y, saved = mul_update_fwd(z, params, direction, eps)
        ctx.direction, ctx.eps = direction, eps
        ctx.save_for_backward(z, saved, *plist)
        return y

    @staticmethod
    def backward(ctx, dy):
        z, saved, *plist = ctx.saved_tensors
        params = dict(zip(MUL_UPDATE_PARAMS, plist))
        dz, grads = mul_update_bwd(z, params, saved, dy.contiguous(), ctx.direction, ctx.eps)
        return (dz, None, None) + tuple(grads[n].to(params[n].dtype) for n in MUL_UPDATE_PARAMS)


def triangle_multiplicative_update(z, params: dict, direction: int = OUTGOING,
                                   eps: float = 1e-5) -> torch.Tensor:
    """Differentiable full triangle multiplicative update (see mul_update_fwd)."""
    return TriangleMultiplicativeUpdate.apply(z, direction, eps,
                                              *[params[n] for n in MUL_UPDATE_PARAMS])


# ------------------------------------------------ LayerNorm and projections --

def proj_problem(z_or_y: torch.Tensor, H: int, c: int, eps: float = 1e-5) -> ProjProblem:
    """Problem of a pair tensor [N, N, cz] or [B, N, N, cz] (rows = N*N per batch
    element)."""
    if z_or_y.dim() not in (3, 4) or z_or_y.shape[-3] != z_or_y.shape[-2]:
        raise ValueError("pair tensors are [N, N, cz] or [B, N, N, cz]")
    B = z_or_y.shape[0] if z_or_y.dim() == 4 else 1
    N, cz = z_or_y.shape[-2], z_or_y.shape[-1]
    return ProjProblem(N * N, B, cz, H, c, eps, 0)


def proj_workspace_size(prob: ProjProblem) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().tri_proj_workspace_size(ctypes.byref(prob), ctypes.byref(n)),
           "tri_proj_workspace_size")
    return n.value


def _proj_ws(prob, ws, device):
    return ws if ws is not None else workspace(proj_workspace_size(prob), device)


def proj_in_fwd(z, gamma, beta, w_qkvg, b_g, w_b, eps: float = 1e-5, outs=None, ws=None,
                stream=None) -> tuple:
    """LayerNorm of the pair representation z ([N, N, cz] or [B, N, N, cz], bf16)
    and its projections: returns (x, stats, q, k, v, g, bias) with x like z,
    stats float32 [.., N, N, 2], q/k/v/g [.., N, N, H, c] bf16 (g: gate logits),
    bias [.., H, N, N] bf16. w_qkvg [cz, 4*H*c] bf16; b_g [H*c] and gamma, beta
    [cz] float32; w_b [cz, H] bf16."""
    H = w_b.shape[1]
    c = w_qkvg.shape[1] // (4 * H)
    prob = proj_problem(z, H, c, eps)
    lead = z.shape[:-1]
    if outs is None:
        x = torch.empty_like(z)
        stats = torch.empty(lead + (2,), dtype=torch.float32, device=z.device)
        q, k, v, g = (torch.empty(lead + (H, c), dtype=z.dtype, device=z.device)
                      for _ in range(4))
        bias = torch.empty(lead[:-2] + (H,) + lead[-2:], dtype=z.dtype, device=z.device)
        outs = (x, stats, q, k, v, g, bias)
    _contig(z, gamma, beta, w_qkvg, b_g, w_b, *outs)
    ws = _proj_ws(prob, ws, z.device)
    _check(lib().tri_proj_in_fwd(ctypes.byref(prob), _p(z), _p(gamma), _p(beta), _p(w_qkvg),
                                 _p(b_g), _p(w_b), *map(_p, outs), _p(ws), ws.numel(),
                                 _stream(stream)), "tri_proj_in_fwd")
    return outs


def proj_in_bwd(z, gamma, w_qkvg, w_b, x, stats, dq, dk, dv, dg, dbias, eps: float = 1e-5,
                grads=None, ws=None, stream=None) -> tuple:
    """(dz, dgamma, dbeta, dw_qkvg, db_g, dw_b) of the input side, given the
    gradients of q, k, v, g and bias; x and stats as proj_in_fwd returned them.
    Parameter gradients are float32 with their parameter's shape."""
    H = w_b.shape[1]
    c = w_qkvg.shape[1] // (4 * H)
    prob = proj_problem(z, H, c, eps)
    if grads is None:
        f32 = dict(dtype=torch.float32, device=z.device)
        grads = (torch.empty_like(z), torch.empty(gamma.shape, **f32),
                 torch.empty(gamma.shape, **f32), torch.empty(w_qkvg.shape, **f32),
                 torch.empty((H * c,), **f32), torch.empty(w_b.shape, **f32))
    _contig(z, gamma, w_qkvg, w_b, x, stats, dq, dk, dv, dg, dbias, *grads)
    ws = _proj_ws(prob, ws, z.device)
    _check(lib().tri_proj_in_bwd(ctypes.byref(prob), _p(z), _p(gamma), _p(w_qkvg), _p(w_b),
                                 _p(x), _p(stats), _p(dq), _p(dk), _p(dv), _p(dg), _p(dbias),
                                 *map(_p, grads), _p(ws), ws.numel(), _stream(stream)),
           "tri_proj_in_bwd")
    return grads


def proj_out_fwd(o, w_o, b_o, y=None, ws=None, stream=None) -> torch.Tensor:
    """y = o w_o + b_o: o [.., N, N, H, c] bf16 (the attention output), w_o
    [H*c, cz] bf16, b_o [cz] float32; y [.., N, N, cz] bf16."""
    H, c = o.shape[-2], o.shape[-1]
    cz = w_o.shape[1]
    if y is None:
        y = torch.empty(o.shape[:-2] + (cz,), dtype=o.dtype, device=o.device)
    prob = proj_problem(y, H, c)
    _contig(o, w_o, b_o, y)
    ws = _proj_ws(prob, ws, o.device)
    _check(lib().tri_proj_out_fwd(ctypes.byref(prob), _p(o), _p(w_o), _p(b_o), _p(y), _p(ws),
                                  ws.numel(), _stream(stream)), "tri_proj_out_fwd")
    return y


def proj_out_bwd(o, w_o, dy, grads=None, ws=None, stream=None) -> tuple:
    """(do, dw_o, db_o) of L = sum(dy * y) for y = proj_out_fwd(o, w_o, b_o)."""
    H, c = o.shape[-2], o.shape[-1]
    prob = proj_problem(dy, H, c)
    if grads is None:
        f32 = dict(dtype=torch.float32, device=o.device)
        grads = (torch.empty_like(o), torch.empty(w_o.shape, **f32),
                 torch.empty((w_o.shape[1],), **f32))
    _contig(o, w_o, dy, *grads)
    ws = _proj_ws(prob, ws, o.device)
    _check(lib().tri_proj_out_bwd(ctypes.byref(prob), _p(o), _p(w_o), _p(dy), *map(_p, grads),
                                  _p(ws), ws.numel(), _stream(stream)), "tri_proj_out_bwd")
    return grads


class TriangleAttentionBlock(torch.autograd.Function):
    """y = TriangleAttentionBlock.apply(z, gamma, beta, w_qkvg, b_g, w_b, w_o, b_o,
    mask, variant, eps): LayerNorm, the q/k/v/gate/bias projections, gated
    triangle attention and the output projection; z [N, N, cz] or [B, N, N, cz]
    bf16 -> y like z (the update that is added to z). Every step runs in the
    library; parameter gradients are computed in float32."""

    @staticmethod
    def forward(ctx, z, gamma, beta, w_qkvg, b_g, w_b, w_o, b_o, mask=None, variant=STARTING,
                eps=1e-5):
        z = z.contiguous()
        x, stats, q, k, v, g, bias = proj_in_fwd(z, gamma, beta, w_qkvg, b_g, w_b, eps)
        o, lse = fwd(q, k, v, bias, g, mask, variant)
        y = proj_out_fwd(o, w_o, b_o)
        ctx.eps, ctx.mask, ctx.variant = eps, mask, variant
        ctx.save_for_backward(z, gamma, w_qkvg, w_b, w_o, x, stats, q, k, v, g, bias, o, lse)
        return y

    @staticmethod
    def backward(ctx, dy):
        z, gamma, w_qkvg, w_b, w_o, x, stats, q, k, v, g, bias, o, lse = ctx.saved_tensors
        do, dw_o, db_o = proj_out_bwd(o, w_o, dy.contiguous())
        dq, dk, dv, dbias, dg = bwd(q, k, v, bias, g, ctx.mask, o, lse, do, ctx.variant)
        dz, dgamma, dbeta, dw_qkvg, db_g, dw_b = proj_in_bwd(z, gamma, w_qkvg, w_b, x, stats, dq,
                                                             dk, dv, dg, dbias, ctx.eps)
        return dz, dgamma, dbeta, dw_qkvg, db_g, dw_b, dw_o, db_o, None, None, None


def triangle_attention_block(z, gamma, beta, w_qkvg, b_g, w_b, w_o, b_o, mask=None,
                             variant: int = STARTING, eps: float = 1e-5) -> torch.Tensor:
    """Differentiable LayerNorm -> projections -> gated triangle attention ->
    output projection; see TriangleAttentionBlock."""
    return TriangleAttentionBlock.apply(z, gamma, beta, w_qkvg, b_g, w_b, w_o, b_o, mask,
                                        variant, eps)
