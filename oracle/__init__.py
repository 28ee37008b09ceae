"""CPU oracle for RQ-LUT logits serving (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never loads it
and shares no code with it.

The arithmetic lives in ``rq_oracle.c`` (plain loops, fp64 and fp32 forms,
compiled with ``-O2 -ffp-contract=off`` and no fast-math).  This module only
compiles it, loads it with ctypes and marshals numpy arrays.

Definitions (pages: "Gemma-2 runtime compression: NF4 + LUT serving", LUT
serving section and correctness-check table; "Gemma-2-2B combined RQ+NF4",
RQ shape paragraph):

* ``lut_build``:  T[b,m,l,k] = sum_j h[b, m*ds+j] * C[m,l,k,j]
* ``logits_lut``: z[b,v] = sum_m sum_l T[b,m,l,code[v,m,l]]
* ``logits_direct``: decode E[v] = sum_l C[m,l,code[v,m,l],:] per subspace,
  then z[b,v] = <h[b], E[v]>  (the pages' reference for their LUT check)
* ``softcap``: y = cap * tanh(z / cap)  (Gemma-2 final-logit softcap, cap 30)
* ``argmax``: lowest index of the maximum
* ``decode_rows_bf16``: bf16_rne(fp32(fp32(sum_l C[m,l,c_l,j]) * scale))
* ``pack10`` / ``unpack10``: 10-bit codes, little-endian bit stream per row
* ``topk``: the k largest values, descending, lower index first on ties
* ``philox4x64_10`` / ``uniform``: the counter-based generator of the
  sampler, u = (word0 >> 11) * 2^-53 for counter (step, row, 0, 0), key
  (seed, 0)
* ``sample_position``: inverse CDF of the temperature softmax over the
  sorted top-k (fp64): first i with running sum > u * total
* ``encode``: greedy residual nearest-codeword codes of rows X (per subspace,
  level by level, fp32 squared distances accumulated with fma in dimension
  order, lowest index on ties, fp32 residual update)
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rq_oracle.c")
_LIB = os.path.join(_HERE, "librq_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C99, no FMA contraction; OpenMP
    splits the row loops across host threads without changing any result)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_f = ctypes.c_float
_d = ctypes.c_double


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    sig = {
        "rqo_lut_build_f64": (None, [_p, _i, _p, _i, _i, _i, _i, _p]),
        "rqo_lut_build_f32": (None, [_p, _i, _p, _i, _i, _i, _i, _p]),
        "rqo_logits_lut_f64": (None, [_p, _i64, _i, _i, _i, _p, _i, _p, _i64, _p]),
        "rqo_logits_lut_f32": (None, [_p, _i64, _i, _i, _i, _p, _i, _p, _i64, _p]),
        "rqo_logits_direct_f64": (None, [_p, _i64, _p, _i, _i, _i, _i, _p, _i, _p, _i64, _p]),
        "rqo_logits_direct_f32": (None, [_p, _i64, _p, _i, _i, _i, _i, _p, _i, _p, _i64, _p]),
        "rqo_softcap_f64": (None, [_p, _i64, _d]),
        "rqo_argmax_f32": (_i64, [_p, _i64]),
        "rqo_argmax_f64": (_i64, [_p, _i64]),
        "rqo_f32_to_bf16_rne": (ctypes.c_uint16, [_f]),
        "rqo_decode_rows_bf16": (None, [_p, _i64, _p, _i64, _p, _i, _i, _i, _i, _f, _p]),
        "rqo_packed10_row_bytes": (_i64, [_i]),
        "rqo_pack10": (None, [_p, _i64, _i, _p]),
        "rqo_unpack10": (None, [_p, _i64, _i, _p]),
        "rqo_encode_f32": (None, [_p, _i64, _p, _i, _i, _i, _i, _p]),
        "rqo_philox4x64_10": (None, [_p, _p, _p]),
        "rqo_uniform": (_d, [ctypes.c_uint64, ctypes.c_uint64, _i64]),
        "rqo_topk_f32": (None, [_p, _i64, _i, _p, _p, _p]),
        "rqo_sample_position": (_i, [_p, _i, _d, _d]),
        "rqo_set_threads": (None, [_i]),
        "rqo_max_threads": (_i, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def set_threads(n: int) -> int:
    """Host threads of the row loops (n < 1: all); returns the count now in
    use.  Results are the same for every count."""
    lib = _load()
    lib.rqo_set_threads(int(n))
    return int(lib.rqo_max_threads())


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dims(C: np.ndarray):
    M, L, K, ds = C.shape
    return M, L, K, ds


def lut_build(h: np.ndarray, C: np.ndarray, precision: str = "f64") -> np.ndarray:
    """T[b, m, l, k] (float64 or float32), h [B, D], C [M, L, K, ds]."""
    lib = _load()
    h = _c(np.atleast_2d(h), np.float32)
    C = _c(C, np.float32)
    M, L, K, ds = _dims(C)
    B, D = h.shape
    assert D == M * ds
    dt = np.float64 if precision == "f64" else np.float32
    T = np.empty((B, M, L, K), dtype=dt)
    fn = lib.rqo_lut_build_f64 if precision == "f64" else lib.rqo_lut_build_f32
    fn(_ptr(h), B, _ptr(C), D, M, L, K, _ptr(T))
    return T


def _rows(rows, V):
    if rows is None:
        rows = np.arange(V, dtype=np.int64)
    return _c(rows, np.int64)


def logits_lut(codes: np.ndarray, T: np.ndarray, rows=None) -> np.ndarray:
    """z[b, r] = sum_m sum_l T[b, m, l, codes[rows[r], m, l]]."""
    lib = _load()
    codes = _c(codes, np.uint16)
    V, M, L = codes.shape
    B, M2, L2, K = T.shape
    assert (M2, L2) == (M, L)
    rows = _rows(rows, V)
    if T.dtype == np.float64:
        z = np.empty((B, rows.size), np.float64)
        lib.rqo_logits_lut_f64(_ptr(codes), V, M, L, K, _ptr(_c(T, np.float64)), B,
                               _ptr(rows), rows.size, _ptr(z))
    else:
        z = np.empty((B, rows.size), np.float32)
        lib.rqo_logits_lut_f32(_ptr(codes), V, M, L, K, _ptr(_c(T, np.float32)), B,
                               _ptr(rows), rows.size, _ptr(z))
    return z


def logits_direct(codes: np.ndarray, C: np.ndarray, h: np.ndarray, rows=None,
                  precision: str = "f64") -> np.ndarray:
    """z[b, r] = <h[b], E[rows[r]]> with E decoded from codes and C."""
    lib = _load()
    codes = _c(codes, np.uint16)
    C = _c(C, np.float32)
    h = _c(np.atleast_2d(h), np.float32)
    V, M, L = codes.shape
    M2, L2, K, ds = C.shape
    B, D = h.shape
    assert (M2, L2) == (M, L) and D == M * ds
    rows = _rows(rows, V)
    if precision == "f64":
        z = np.empty((B, rows.size), np.float64)
        lib.rqo_logits_direct_f64(_ptr(codes), V, _ptr(C), D, M, L, K, _ptr(h), B,
                                  _ptr(rows), rows.size, _ptr(z))
    else:
        z = np.empty((B, rows.size), np.float32)
        lib.rqo_logits_direct_f32(_ptr(codes), V, _ptr(C), D, M, L, K, _ptr(h), B,
                                  _ptr(rows), rows.size, _ptr(z))
    return z


def softcap(z: np.ndarray, cap: float) -> np.ndarray:
    """y = cap * tanh(z / cap) in fp64 (cap <= 0: identity)."""
    lib = _load()
    y = np.array(z, dtype=np.float64, copy=True, order="C")
    lib.rqo_softcap_f64(_ptr(y), y.size, float(cap))
    return y


def argmax(y: np.ndarray) -> np.ndarray:
    """Per-token lowest index of the maximum; y [B, n] float32 or float64."""
    lib = _load()
    y2 = np.atleast_2d(y)
    out = np.empty(y2.shape[0], np.int64)
    for b in range(y2.shape[0]):
        if y2.dtype == np.float64:
            row = _c(y2[b], np.float64)
            out[b] = lib.rqo_argmax_f64(_ptr(row), row.size)
        else:
            row = _c(y2[b], np.float32)
            out[b] = lib.rqo_argmax_f32(_ptr(row), row.size)
    return out


def f32_to_bf16_rne(x: float) -> int:
    return int(_load().rqo_f32_to_bf16_rne(float(np.float32(x))))


def decode_rows_bf16(ids: np.ndarray, codes: np.ndarray, C: np.ndarray,
                     scale: float) -> np.ndarray:
    """bf16 bit patterns (uint16) [N, D] of the rebuilt input rows."""
    lib = _load()
    ids = _c(ids, np.int32)
    codes = _c(codes, np.uint16)
    C = _c(C, np.float32)
    V, M, L = codes.shape
    M2, L2, K, ds = C.shape
    assert (M2, L2) == (M, L)
    D = M * ds
    out = np.empty((ids.size, D), np.uint16)
    lib.rqo_decode_rows_bf16(_ptr(ids), ids.size, _ptr(codes), V, _ptr(C), D, M, L,
                             K, float(scale), _ptr(out))
    return out


def packed10_row_bytes(P: int) -> int:
    return int(_load().rqo_packed10_row_bytes(P))


def pack10(codes: np.ndarray) -> np.ndarray:
    """codes uint16 [V, P] or [V, M, L] (all < 1024) -> uint8 [V, row_bytes]."""
    lib = _load()
    codes = _c(codes, np.uint16)
    V = codes.shape[0]
    P = int(np.prod(codes.shape[1:]))
    rb = packed10_row_bytes(P)
    out = np.empty((V, rb), np.uint8)
    lib.rqo_pack10(_ptr(codes), V, P, _ptr(out))
    return out


def unpack10(packed: np.ndarray, P: int) -> np.ndarray:
    lib = _load()
    packed = _c(packed, np.uint8)
    V = packed.shape[0]
    assert packed.shape[1] == packed10_row_bytes(P)
    out = np.empty((V, P), np.uint16)
    lib.rqo_unpack10(_ptr(packed), V, P, _ptr(out))
    return out


def encode(X: np.ndarray, C: np.ndarray) -> np.ndarray:
    """codes uint16 [N, M, L] of rows X [N, D] against codebooks C [M, L, K, ds]."""
    lib = _load()
    X = _c(np.atleast_2d(X), np.float32)
    C = _c(C, np.float32)
    M, L, K, ds = _dims(C)
    N, D = X.shape
    assert D == M * ds and ds <= 64 and K <= 65536
    out = np.empty((N, M, L), np.uint16)
    lib.rqo_encode_f32(_ptr(X), N, _ptr(C), D, M, L, K, _ptr(out))
    return out


def philox4x64_10(ctr, key) -> np.ndarray:
    lib = _load()
    c = _c(np.asarray(ctr, dtype=np.uint64), np.uint64)
    k = _c(np.asarray(key, dtype=np.uint64), np.uint64)
    out = np.empty(4, np.uint64)
    lib.rqo_philox4x64_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def uniform(seed: int, step: int, row: int) -> float:
    return float(_load().rqo_uniform(seed, step, row))


def topk(y: np.ndarray, k: int):
    """(values float32 [B, k], indices int32 [B, k]) of y [B, n] float32."""
    lib = _load()
    y2 = np.atleast_2d(_c(y, np.float32))
    B, n = y2.shape
    val = np.empty((B, k), np.float32)
    idx = np.empty((B, k), np.int32)
    taken = np.empty(n, np.uint8)
    for b in range(B):
        row = np.ascontiguousarray(y2[b])
        vb = np.empty(k, np.float32)
        ib = np.empty(k, np.int32)
        lib.rqo_topk_f32(_ptr(row), n, k, _ptr(vb), _ptr(ib), _ptr(taken))
        val[b], idx[b] = vb, ib
    return val, idx


def sample_position(val: np.ndarray, temperature: float, u: float) -> int:
    v = _c(val, np.float32)
    return int(_load().rqo_sample_position(_ptr(v), v.size, float(temperature), float(u)))


def sample(y: np.ndarray, k: int, temperature: float, seed: int, step: int):
    """Top-k values/indices and the sampled token of every row of y [B, n]."""
    val, idx = topk(y, k)
    tok = np.array([idx[b, sample_position(val[b], temperature, uniform(seed, step, b))]
                    for b in range(val.shape[0])], np.int32)
    return val, idx, tok


def reference_logits(codes: np.ndarray, C: np.ndarray, h: np.ndarray, cap: float,
                     rows=None):
    """Parity reference: fp64 LUT logits, softcapped in fp64.

    Returns (y64 [B, n] float64, y32 = y64 rounded to float32)."""
    T = lut_build(h, C, "f64")
    z = logits_lut(codes, T, rows)
    y = softcap(z, cap)
    return y, y.astype(np.float32)
