"""librqlut Python binding: LUT-based serving of a residual-product-quantized
(RQ) tied embedding on one B200.

Thin ctypes marshalling over the C ABI declared in ``include/rqlut.h``; every
step of the computation runs in the library's sm_100a CUDA kernels.  PyTorch
only provides device memory and the current stream.  The functions keep the C
names:

* ``rq_lut_build``  -- per-token tables T[p][k][b] = <h_b[m], C[m][l][k]>
* ``rq_lut_logits`` -- z[b][v] = sum_p T[p][code[v][p]][b], softcap, argmax
* ``rq_logits_from_hidden`` -- both, large batches in token groups of 32;
  a full group's rows are decoded and multiplied on the tensor cores
  (``rq_logits_from_hidden_path`` picks tables, FP32 or tensor cores)
* ``rq_decode_rows`` -- bf16 input rows rebuilt on demand
* ``rq_pack10`` -- uint16 codes -> 10-bit packed rows
* ``rq_prepare_sched``, ``rq_prepare_rot10`` -- the batch-1 layouts of
  uint16 and 10-bit codes (bank-scheduled, rotated slices)

(method: "Gemma-2 runtime compression: NF4 + LUT serving", LUT section.)
There is no CPU fallback: if the library or a GPU is missing, calls raise.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

__all__ = [
    "RqDims", "RqError", "U16", "PACKED10", "SCHED", "U8", "ROT10", "lib", "rq_pack8", "dims",
    "rq_prepare_sched", "rq_prepare_rot10",
    "rq_status_string", "rq_version", "rq_codes_bytes", "rq_lut_token_stride",
    "rq_lut_bytes", "rq_logits_workspace_bytes", "rq_fused_workspace_bytes",
    "rq_lut_build", "rq_lut_logits", "rq_logits_from_hidden", "rq_logits_from_hidden_path",
    "rq_decode_rows",
    "rq_pack10", "rq_device_error", "rq_set_profile_events", "rq_lut_logits_static",
    "rq_greedy_step", "rq_encode", "rq_topk_workspace_bytes", "rq_topk_sample",
    "rq_last_cuda_error", "rq_cuda_error_name", "PATH_AUTO", "PATH_TABLES", "PATH_DECODE_FP32",
    "PATH_DECODE_TC", "rq_argmax_candidates", "rq_argmax_merge", "shard_rows", "rq_sharded_logits",
]

U16 = 0
PACKED10 = 1
SCHED = 2
U8 = 3
ROT10 = 4        # RQ_CODES_PACKED10_ROT
# kernel of full 32-token groups in rq_logits_from_hidden (rqlut.h RQ_PATH_*)
PATH_AUTO = 0
PATH_TABLES = 1
PATH_DECODE_FP32 = 2
PATH_DECODE_TC = 3

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librqlut.so")


class RqDims(ctypes.Structure):
    _fields_ = [("V", ctypes.c_int64), ("D", ctypes.c_int32), ("M", ctypes.c_int32),
                ("L", ctypes.c_int32), ("K", ctypes.c_int32)]

    def __repr__(self):
        return f"RqDims(V={self.V}, D={self.D}, M={self.M}, L={self.L}, K={self.K})"


def dims(V, D, M, L, K) -> RqDims:
    return RqDims(int(V), int(D), int(M), int(L), int(K))


class RqError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        msg = f"{fn} failed: {rq_status_string(status)} ({status})"
        if status == 4:   # RQ_ERR_CUDA: name the runtime error behind it
            err = rq_last_cuda_error(clear=True)
            msg += f" [{rq_cuda_error_name(err)}]"
        super().__init__(msg)


_lib = None
_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t
_f = ctypes.c_float

_SIGNATURES = {
    "rq_status_string": (ctypes.c_char_p, [_i]),
    "rq_version": (_i, []),
    "rq_codes_bytes": (_sz, [RqDims, _i]),
    "rq_lut_token_stride": (_i, [_i]),
    "rq_lut_bytes": (_sz, [RqDims, _i]),
    "rq_logits_workspace_bytes": (_sz, [RqDims, _i, _i, _i]),
    "rq_fused_workspace_bytes": (_sz, [RqDims, _i, _i, _i]),
    "rq_lut_build": (_i, [_p, _p, RqDims, _i, _p, _p]),
    "rq_lut_logits": (_i, [_p, _i, RqDims, _p, _i, _f, _p, _p, _p, _sz, _p]),
    "rq_logits_from_hidden": (_i, [_p, _p, _p, _i, RqDims, _i, _f, _p, _p, _p, _sz, _p]),
    "rq_logits_from_hidden_path": (_i, [_p, _p, _p, _i, RqDims, _i, _f, _p, _p, _p, _sz, _i,
                                        _p]),
    "rq_decode_rows": (_i, [_p, _i64, _p, _i, _p, RqDims, _f, _p, _p]),
    "rq_pack10": (_i, [_p, RqDims, _p, _p]),
    "rq_pack8": (_i, [_p, RqDims, _p, _p]),
    "rq_encode": (_i, [_p, RqDims, _p, _p, _p]),
    "rq_topk_workspace_bytes": (_sz, [_i64, _i, _i]),
    "rq_last_cuda_error": (_i, [_i]),
    "rq_cuda_error_name": (ctypes.c_char_p, [_i]),
    "rq_topk_sample": (_i, [_p, _i64, _i, _i, _f, ctypes.c_uint64, ctypes.c_uint64, _p, _p, _p,
                            _p, _sz, _p]),
    "rq_device_error": (_i, [ctypes.POINTER(ctypes.c_uint32), _i]),
    "rq_set_profile_events": (_i, [_p, _p]),
    "rq_prepare_sched": (_i, [_p, RqDims, _p, _p, _p]),
    "rq_prepare_rot10": (_i, [_p, RqDims, _p, _p, _p]),
    "rq_lut_logits_static": (_i, [_p, _i, RqDims, _p, _i, _f, _p, _p, _p]),
    "rq_greedy_step": (_i, [_p, _p, _p, _i, RqDims, _i, _f, _p, _p, _f, _p, _p, _sz, _p]),
    "rq_argmax_candidates": (_i, [_p, _p, _i, _i64, _i64, _p, _p, _p]),
    "rq_argmax_merge": (_i, [_p, _p, _i, _i, _p, _p]),
}


def lib() -> ctypes.CDLL:
    """Load librqlut.so (built in-tree by ``lut_logits_serving_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"librqlut.so not found at {LIB_PATH}; build it with "
                "`python -m lut_logits_serving_b200.build` (there is no CPU fallback)")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


# ------------------------------------------------------------ host queries

def rq_status_string(status: int) -> str:
    return lib().rq_status_string(int(status)).decode()


def rq_version() -> int:
    return lib().rq_version()


def rq_codes_bytes(d: RqDims, fmt: int) -> int:
    return lib().rq_codes_bytes(d, fmt)


def rq_lut_token_stride(B: int) -> int:
    return lib().rq_lut_token_stride(B)


def rq_lut_bytes(d: RqDims, B: int) -> int:
    return lib().rq_lut_bytes(d, B)


def rq_logits_workspace_bytes(d: RqDims, B: int, fmt: int, want_argmax: bool) -> int:
    return lib().rq_logits_workspace_bytes(d, B, fmt, int(bool(want_argmax)))


def rq_fused_workspace_bytes(d: RqDims, B: int, fmt: int, want_argmax: bool) -> int:
    return lib().rq_fused_workspace_bytes(d, B, fmt, int(bool(want_argmax)))


# ------------------------------------------------------------ device calls

def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _cuda(t, dtype, name, nbytes=None):
    """Device pointer of `t` after checking its type, layout and, with
    `nbytes`, that it holds at least that many bytes: the C calls take bare
    pointers, so a short buffer would otherwise be read or written past its
    end."""
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name}: expected a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if nbytes is not None and t.numel() * t.element_size() < nbytes:
        raise ValueError(f"{name}: {t.numel() * t.element_size()} bytes, "
                         f"the call needs {nbytes}")
    if not _on_device(t):
        raise ValueError(f"{name}: must be a CUDA tensor (no CPU fallback)")
    return ctypes.c_void_p(t.data_ptr())


def _on_device(t):
    return t.is_cuda


def _ptr_or_null(t, dtype, name, nbytes=None):
    return ctypes.c_void_p(None) if t is None else _cuda(t, dtype, name, nbytes)


def _book_bytes(d):
    """Bytes of the codebooks C [M, L, K, ds] (fp32)."""
    return d.M * d.L * d.K * (d.D // d.M if d.M > 0 else 0) * 4


def _tokens(h, d, name="h"):
    """B of hidden states h [B, D] (or [D] for one token)."""
    if h.dim() == 1 and h.shape[0] == d.D:
        return 1
    if h.dim() != 2 or h.shape[1] != d.D:
        raise ValueError(f"{name}: shape {tuple(h.shape)}, expected [B, {d.D}]")
    return h.shape[0]


def _check(fn, status):
    if status != 0:
        raise RqError(fn, status)


def _codes_dtype(fmt):
    torch = _torch()
    return torch.uint8 if fmt in (PACKED10, U8, ROT10) else torch.uint16


def _empty(shape, dtype, like):
    torch = _torch()
    return torch.empty(shape, dtype=dtype, device=like.device)


def _workspace(nbytes, like, ws):
    torch = _torch()
    if nbytes == 0:
        return ctypes.c_void_p(None), 0, ws
    if ws is None or ws.numel() * ws.element_size() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=like.device)
    return _cuda(ws, None, "ws"), ws.numel() * ws.element_size(), ws


def rq_lut_build(h, C, d: RqDims, lut=None, stream=None):
    """h float32 [B, D], C float32 [M, L, K, ds] -> lut float32 [P, K, Bs]."""
    torch = _torch()
    B = _tokens(h, d)
    Bs = rq_lut_token_stride(B)
    if lut is None:
        lut = _empty((d.M * d.L, d.K, Bs), torch.float32, h)
    _check("rq_lut_build", lib().rq_lut_build(
        _cuda(h, torch.float32, "h"), _cuda(C, torch.float32, "C", _book_bytes(d)), d, B,
        _cuda(lut, torch.float32, "lut", rq_lut_bytes(d, B)), _stream(stream)))
    return lut


def rq_lut_logits(codes, fmt: int, d: RqDims, lut, B: int, softcap: float = 30.0,
                  want_logits: bool = True, want_argmax: bool = False, logits=None,
                  argmax=None, ws=None, stream=None):
    """Returns (logits float32 [B, V] or None, argmax int32 [B] or None, ws)."""
    torch = _torch()
    if want_logits and logits is None:
        logits = _empty((B, d.V), torch.float32, lut)
    if want_argmax and argmax is None:
        argmax = _empty((B,), torch.int32, lut)
    nbytes = rq_logits_workspace_bytes(d, B, fmt, argmax is not None)
    wp, wn, ws = _workspace(nbytes, lut, ws)
    _check("rq_lut_logits", lib().rq_lut_logits(
        _cuda(codes, _codes_dtype(fmt), "codes", rq_codes_bytes(d, fmt)), fmt, d,
        _cuda(lut, torch.float32, "lut", rq_lut_bytes(d, B)), B,
        float(softcap), _ptr_or_null(logits, torch.float32, "logits", B * d.V * 4),
        _ptr_or_null(argmax, torch.int32, "argmax", B * 4), wp, wn, _stream(stream)))
    return logits, argmax, ws


def rq_logits_from_hidden(h, C, codes, fmt: int, d: RqDims, softcap: float = 30.0,
                          want_logits: bool = True, want_argmax: bool = False, logits=None,
                          argmax=None, ws=None, stream=None, path: int = None):
    """Returns (logits float32 [B, V] or None, argmax int32 [B] or None, ws).
    ``path`` (one of PATH_*) picks the kernel of full 32-token groups; None
    is the library's default (rq_logits_from_hidden)."""
    torch = _torch()
    B = _tokens(h, d)
    if want_logits and logits is None:
        logits = _empty((B, d.V), torch.float32, h)
    if want_argmax and argmax is None:
        argmax = _empty((B,), torch.int32, h)
    nbytes = rq_fused_workspace_bytes(d, B, fmt, argmax is not None)
    wp, wn, ws = _workspace(nbytes, h, ws)
    args = (_cuda(h, torch.float32, "h"), _cuda(C, torch.float32, "C", _book_bytes(d)),
            _cuda(codes, _codes_dtype(fmt), "codes", rq_codes_bytes(d, fmt)), fmt, d, B,
            float(softcap), _ptr_or_null(logits, torch.float32, "logits", B * d.V * 4),
            _ptr_or_null(argmax, torch.int32, "argmax", B * 4), wp, wn)
    if path is None:
        _check("rq_logits_from_hidden", lib().rq_logits_from_hidden(*args, _stream(stream)))
    else:
        _check("rq_logits_from_hidden_path",
               lib().rq_logits_from_hidden_path(*args, int(path), _stream(stream)))
    return logits, argmax, ws


def rq_logits_from_hidden_path(h, C, codes, fmt: int, d: RqDims, path: int,
                               softcap: float = 30.0, **kw):
    """rq_logits_from_hidden with an explicit kernel for full token groups."""
    return rq_logits_from_hidden(h, C, codes, fmt, d, softcap, path=path, **kw)


def rq_argmax_candidates(logits, argmax, row0: int, val=None, gidx=None, stream=None):
    """A vocabulary shard's winner per token: (value float32 [B], global row
    int32 [B]) from its logits [B, V_shard] and argmax [B]."""
    torch = _torch()
    if logits.dim() != 2:
        raise ValueError("logits: [B, V_shard] expected")
    B, V = logits.shape
    if val is None:
        val = _empty((B,), torch.float32, logits)
    if gidx is None:
        gidx = _empty((B,), torch.int32, logits)
    _check("rq_argmax_candidates", lib().rq_argmax_candidates(
        _cuda(logits, torch.float32, "logits"), _cuda(argmax, torch.int32, "argmax", B * 4),
        B, V, int(row0), _cuda(val, torch.float32, "val", B * 4),
        _cuda(gidx, torch.int32, "gidx", B * 4), _stream(stream)))
    return val, gidx


def rq_argmax_merge(val, gidx, out=None, stream=None):
    """Global argmax int32 [B] from n shards' candidates val, gidx [n, B]."""
    torch = _torch()
    if val.dim() != 2 or tuple(gidx.shape) != tuple(val.shape):
        raise ValueError("val, gidx: [n, B] expected")
    n, B = val.shape
    if out is None:
        out = _empty((B,), torch.int32, val)
    _check("rq_argmax_merge", lib().rq_argmax_merge(
        _cuda(val, torch.float32, "val"), _cuda(gidx, torch.int32, "gidx"), n, B,
        _cuda(out, torch.int32, "argmax", B * 4), _stream(stream)))
    return out


def shard_rows(V: int, rank: int, world: int):
    """Rows [row0, row1) of vocabulary shard `rank` of `world` (even split)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank, world")
    return V * rank // world, V * (rank + 1) // world


def rq_sharded_logits(h, C, codes_shard, fmt: int, d_shard: RqDims, row0: int,
                      softcap: float = 30.0, group=None, ws=None, stream=None):
    """Logits of this rank's vocabulary rows and the global greedy pick: the
    fused call on the shard, its per-token winner, one all-gather of the
    winners over the process group (NCCL), and the merge.  Returns (logits
    [B, V_shard], argmax int32 [B] of global rows, ws)."""
    torch = _torch()
    logits, am, ws = rq_logits_from_hidden(h, C, codes_shard, fmt, d_shard, softcap,
                                           want_argmax=True, ws=ws, stream=stream)
    val, gidx = rq_argmax_candidates(logits, am, row0, stream=stream)
    world = 1
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        world = dist.get_world_size(group)
    if world > 1:
        # flat [world * B] buffers, rank-major (the layout every backend takes);
        # the collectives are ordered after the candidates on the call's stream
        vals = _empty((world * val.numel(),), torch.float32, val)
        idxs = _empty((world * gidx.numel(),), torch.int32, gidx)
        with torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext():
            dist.all_gather_into_tensor(vals, val, group=group)
            dist.all_gather_into_tensor(idxs, gidx, group=group)
        vals, idxs = vals.view(world, -1), idxs.view(world, -1)
    else:
        vals, idxs = val.view(1, -1), gidx.view(1, -1)
    return logits, rq_argmax_merge(vals, idxs, stream=stream), ws


def rq_decode_rows(ids, codes, fmt: int, C, d: RqDims, scale: float, out=None, stream=None):
    """ids int32 [N] -> bf16 rows [N, D] (returned as torch.bfloat16)."""
    torch = _torch()
    N = ids.numel()
    if out is None:
        out = _empty((N, d.D), torch.bfloat16, ids)
    if out.dtype not in (torch.bfloat16, torch.uint16, torch.int16):
        raise ValueError("out: bf16 rows expected")
    _check("rq_decode_rows", lib().rq_decode_rows(
        _cuda(ids, torch.int32, "ids"), N,
        _cuda(codes, _codes_dtype(fmt), "codes", rq_codes_bytes(d, fmt)), fmt,
        _cuda(C, torch.float32, "C", _book_bytes(d)), d, float(scale),
        _cuda(out, None, "out", N * d.D * 2), _stream(stream)))
    return out


def rq_pack10(codes_u16, d: RqDims, out=None, stream=None):
    """uint16 [V, P] (or [V, M, L]) -> uint8 [V, ceil(10 P / 8)]."""
    torch = _torch()
    if out is None:
        out = _empty((d.V, rq_codes_bytes(d, PACKED10) // d.V), torch.uint8, codes_u16)
    _check("rq_pack10", lib().rq_pack10(
        _cuda(codes_u16, torch.uint16, "codes_u16", rq_codes_bytes(d, U16)), d,
        _cuda(out, torch.uint8, "packed", rq_codes_bytes(d, PACKED10)), _stream(stream)))
    return out


def rq_encode(X, C, d: RqDims, out=None, stream=None):
    """Rows float32 [V, D] -> uint16 codes [V, M*L]: greedy residual
    nearest-codeword assignment against C [M, L, K, ds]."""
    torch = _torch()
    if out is None:
        out = _empty((d.V, d.M * d.L), torch.uint16, X)
    _check("rq_encode", lib().rq_encode(
        _cuda(X, torch.float32, "X", d.V * d.D * 4), d,
        _cuda(C, torch.float32, "C", _book_bytes(d)),
        _cuda(out, torch.uint16, "codes", rq_codes_bytes(d, U16)), _stream(stream)))
    return out


def rq_last_cuda_error(clear: bool = False) -> int:
    return int(lib().rq_last_cuda_error(int(bool(clear))))


def rq_cuda_error_name(err: int) -> str:
    return lib().rq_cuda_error_name(int(err)).decode()


def rq_topk_workspace_bytes(V: int, B: int, k: int) -> int:
    return int(lib().rq_topk_workspace_bytes(V, B, k))


def rq_topk_sample(logits, k: int, temperature: float = 1.0, seed: int = 0, step: int = 0,
                   topk_val=None, topk_idx=None, token=None, want_topk: bool = True,
                   ws=None, stream=None):
    """logits float32 [B, V] (device) -> (topk_val [B, k], topk_idx [B, k], token [B]);
    the top-k outputs are None with want_topk=False."""
    torch = _torch()
    if logits.dim() != 2:
        raise ValueError("logits: [B, V] expected")
    B, V = logits.shape
    if want_topk:
        if topk_val is None:
            topk_val = _empty((B, k), torch.float32, logits)
        if topk_idx is None:
            topk_idx = _empty((B, k), torch.int32, logits)
    if token is None:
        token = _empty((B,), torch.int32, logits)
    nbytes = rq_topk_workspace_bytes(V, B, k)
    wsp, wsn, ws = _workspace(max(nbytes, 1), logits, ws)
    _check("rq_topk_sample", lib().rq_topk_sample(
        _cuda(logits, torch.float32, "logits"), V, B, k, float(temperature),
        ctypes.c_uint64(seed), ctypes.c_uint64(step),
        _ptr_or_null(topk_val, torch.float32, "topk_val", B * k * 4),
        _ptr_or_null(topk_idx, torch.int32, "topk_idx", B * k * 4),
        _cuda(token, torch.int32, "token", B * 4), wsp, wsn, _stream(stream)))
    return topk_val, topk_idx, token


def rq_pack8(codes_u16, d: RqDims, out=None, stream=None):
    """uint16 [V, P] (or [V, M, L]) -> uint8 [V, P] (RQ_CODES_U8, K <= 256)."""
    torch = _torch()
    if out is None:
        out = _empty((d.V, d.M * d.L), torch.uint8, codes_u16)
    _check("rq_pack8", lib().rq_pack8(
        _cuda(codes_u16, torch.uint16, "codes_u16", rq_codes_bytes(d, U16)), d,
        _cuda(out, torch.uint8, "packed", rq_codes_bytes(d, U8)), _stream(stream)))
    return out


def rq_device_error(clear: bool = True) -> int:
    v = ctypes.c_uint32(0)
    _check("rq_device_error", lib().rq_device_error(ctypes.byref(v), int(bool(clear))))
    return v.value


def rq_set_profile_events(start=None, stop=None):
    """start/stop: torch.cuda.Event (enable_timing=True) or None to switch off."""
    sp = ctypes.c_void_p(start.cuda_event if start is not None else None)
    tp = ctypes.c_void_p(stop.cuda_event if stop is not None else None)
    _check("rq_set_profile_events", lib().rq_set_profile_events(sp, tp))


def rq_prepare_sched(codes_u16, d: RqDims, out=None, stats=None, stream=None):
    """uint16 codes [V, P] -> bank-scheduled uint16 codes [V, P] (RQ_CODES_SCHED).
    With stats=True returns (out, (steps, bank passes)) after a sync."""
    torch = _torch()
    if out is None:
        out = torch.empty((d.V, d.M * d.L), dtype=torch.uint16, device=codes_u16.device)
    st = None
    if stats:
        st = torch.zeros(2, dtype=torch.int64, device=codes_u16.device)
    _check("rq_prepare_sched", lib().rq_prepare_sched(
        _cuda(codes_u16, torch.uint16, "codes_u16", rq_codes_bytes(d, U16)), d,
        _cuda(out, torch.uint16, "out", rq_codes_bytes(d, SCHED)),
        _ptr_or_null(st, torch.int64, "stats", 16), _stream(stream)))
    if stats:
        v = st.cpu().tolist()
        return out, (v[0], v[1])
    return out


def rq_prepare_rot10(codes_u16, d: RqDims, out=None, stats=None, stream=None):
    """uint16 codes [V, P] -> RQ_CODES_PACKED10_ROT bytes (rotated 10-bit slices,
    then the rotations).  With stats=True returns (out, (steps, bank passes))
    after a sync."""
    torch = _torch()
    nbytes = rq_codes_bytes(d, ROT10)
    if out is None:
        out = torch.empty((nbytes,), dtype=torch.uint8, device=codes_u16.device)
    st = None
    if stats:
        st = torch.zeros(2, dtype=torch.int64, device=codes_u16.device)
    _check("rq_prepare_rot10", lib().rq_prepare_rot10(
        _cuda(codes_u16, torch.uint16, "codes_u16", rq_codes_bytes(d, U16)), d,
        _cuda(out, torch.uint8, "out", nbytes), _ptr_or_null(st, torch.int64, "stats", 16),
        _stream(stream)))
    if stats:
        v = st.cpu().tolist()
        return out, (v[0], v[1])
    return out


def rq_lut_logits_static(codes, fmt: int, d: RqDims, lut, B: int, softcap: float = 30.0,
                         want_logits: bool = True, want_argmax: bool = False, logits=None,
                         argmax=None, stream=None):
    """rq_lut_logits with the library's fixed device scratch as workspace
    (for callers that cannot allocate; see include/rqlut.h).
    Returns (logits or None, argmax or None)."""
    torch = _torch()
    if want_logits and logits is None:
        logits = _empty((B, d.V), torch.float32, lut)
    if want_argmax and argmax is None:
        argmax = _empty((B,), torch.int32, lut)
    _check("rq_lut_logits_static", lib().rq_lut_logits_static(
        _cuda(codes, _codes_dtype(fmt), "codes", rq_codes_bytes(d, fmt)), fmt, d,
        _cuda(lut, torch.float32, "lut", rq_lut_bytes(d, B)), B,
        float(softcap), _ptr_or_null(logits, torch.float32, "logits", B * d.V * 4),
        _ptr_or_null(argmax, torch.int32, "argmax", B * 4), _stream(stream)))
    return logits, argmax


def rq_greedy_step(h, C, codes, fmt: int, d: RqDims, softcap: float = 30.0, scale: float = 1.0,
                   want_logits: bool = True, logits=None, argmax=None, rows=None, ws=None,
                   stream=None):
    """Logits (optional), argmax and the bf16 input rows of the picked tokens.
    Returns (logits or None, argmax int32 [B], rows bf16 [B, D], ws)."""
    torch = _torch()
    B = _tokens(h, d)
    if want_logits and logits is None:
        logits = _empty((B, d.V), torch.float32, h)
    if argmax is None:
        argmax = _empty((B,), torch.int32, h)
    if rows is None:
        rows = _empty((B, d.D), torch.bfloat16, h)
    nbytes = rq_fused_workspace_bytes(d, B, fmt, True)
    wp, wn, ws = _workspace(nbytes, h, ws)
    _check("rq_greedy_step", lib().rq_greedy_step(
        _cuda(h, torch.float32, "h"), _cuda(C, torch.float32, "C", _book_bytes(d)),
        _cuda(codes, _codes_dtype(fmt), "codes", rq_codes_bytes(d, fmt)), fmt, d, B,
        float(softcap), _ptr_or_null(logits, torch.float32, "logits", B * d.V * 4),
        _cuda(argmax, torch.int32, "argmax", B * 4), float(scale),
        _cuda(rows, None, "rows", B * d.D * 2), wp, wn, _stream(stream)))
    return logits, argmax, rows, ws
