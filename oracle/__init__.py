"""CPU oracle for grouped-query split-KV decode attention (fp64).

TEST INFRASTRUCTURE ONLY: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  The CUDA library never
loads it, and it shares no code with the CUDA library.

The arithmetic lives in ``oracle.c`` (plain C, fp64, two-pass softmax); this
module only compiles it with gcc on first use and marshals arrays through
ctypes.  What it computes is stated in the header of ``oracle.c`` with the
passages of the kernbench "_attention_mesh_mlo.py" page it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-fPIC", "-shared",
             "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Oracle:
    """ctypes handle on one compiled copy of ``oracle.c``."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        vp, i32p, f64p = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_double)
        ci, cd = ctypes.c_int, ctypes.c_double
        lib.oracle_attn.argtypes = [vp, vp, vp, i32p, ci, ci, ci, ci, cd, ci, i32p, ci, ci, f64p]
        lib.oracle_attn.restype = ci
        lib.oracle_partials.argtypes = [vp, vp, vp, i32p, ci, ci, ci, ci, cd, ci, ci, ci, ci,
                                        i32p, ci, ci, f64p, f64p, f64p]
        lib.oracle_partials.restype = ci
        lib.oracle_merge.argtypes = [f64p, f64p, f64p, ci, ci, ci, f64p]
        lib.oracle_merge.restype = None
        lib.oracle_prefill.argtypes = [vp, vp, vp, i32p, ci, ci, ci, ci, cd, ci, i32p, ci, ci, f64p]
        lib.oracle_prefill.restype = ci
        self.lib = lib
        self.path = path

    def attn(self, *a, **kw):
        return _attn(self.lib, *a, **kw)

    def partials(self, *a, **kw):
        return _partials(self.lib, *a, **kw)

    def merge(self, *a, **kw):
        return _merge(self.lib, *a, **kw)

    def prefill(self, *a, **kw):
        return _prefill(self.lib, *a, **kw)


def compile_variant(src_text: str, out_path: str) -> Oracle:
    """Compile a (possibly edited) copy of the oracle source to ``out_path``.

    Used by the tests that plant a mistake in a copy of the oracle and check
    that the pins catch it; the committed source is never modified."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-fPIC", "-shared",
                           "-pthread", "-o", out_path, src, "-lm"])
    return Oracle(out_path)


def source() -> str:
    with open(_SRC) as f:
        return f.read()


def default() -> Oracle:
    global _lib
    with _lock:
        if _lib is None:
            _lib = Oracle(build())
    return _lib


def _raw(x):
    """Contiguous numpy view of a CPU array / tensor plus its dtype code.

    fp32 stays fp32; bf16 is passed as its raw 16-bit patterns."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().contiguous()
            if x.dtype == torch.bfloat16:
                return np.ascontiguousarray(x.view(torch.int16).numpy()), BF16
            if x.dtype == torch.float32:
                return np.ascontiguousarray(x.numpy()), F32
            raise TypeError(f"oracle inputs must be fp32 or bf16, got {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    raise TypeError(f"oracle inputs must be fp32 (or torch bf16), got {x.dtype}")


def _items(B, h_q, items):
    if items is None:
        items = [(b, h) for b in range(B) for h in range(h_q)]
    arr = np.ascontiguousarray(np.asarray(items, dtype=np.int32).reshape(-1, 2))
    return arr


def _ptr(a, t):
    return a.ctypes.data_as(ctypes.POINTER(t))


def attn(*a, **kw):
    return default().attn(*a, **kw)


def partials(*a, **kw):
    return default().partials(*a, **kw)


def merge(*a, **kw):
    return default().merge(*a, **kw)


def prefill(*a, **kw):
    return default().prefill(*a, **kw)


def _prefill(lib, q, k, v, seqlens, h_q: int, h_kv: int, scale: float, items=None, nthreads: int = 0):
    """Causal prefill output in fp64.

    q: packed [sum S_b, h_q, d]; k, v: packed [sum S_b, h_kv, d]; seqlens
    int32 [B].  ``items`` selects (b, h, i) triples -- query position i of
    sequence b, head h (default: all, in (b, i, h) order, i.e. q's row
    order).  Returns float64 [n_items, d]."""
    qa, dt = _raw(q)
    ka, _ = _raw(k)
    va, _ = _raw(v)
    sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    B = sl.shape[0]
    d = qa.shape[-1]
    if items is None:
        items = [(b, h, i) for b in range(B) for i in range(int(sl[b])) for h in range(h_q)]
    it = np.ascontiguousarray(np.asarray(items, dtype=np.int32).reshape(-1, 3))
    out = np.zeros((it.shape[0], d), dtype=np.float64)
    rc = lib.oracle_prefill(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, _ptr(sl, ctypes.c_int32),
                            B, h_q, h_kv, d, float(scale), dt, _ptr(it, ctypes.c_int32), it.shape[0],
                            nthreads, _ptr(out, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle_prefill: bad arguments")
    return out


def _attn(lib, q, k, v, seqlens, h_q: int, h_kv: int, scale: float, items=None, nthreads: int = 0):
    """Exact attention output in fp64.

    q: [B, h_q, d]; k, v: packed [sum S_b, h_kv, d] (fp32 or bf16); seqlens:
    int32 [B].  ``items`` selects (b, h) pairs (default: all, in (b, h)
    order).  Returns float64 [n_items, d]."""
    qa, dt = _raw(q)
    ka, dk = _raw(k)
    va, dv = _raw(v)
    assert dt == dk == dv, "q, k and v must share one dtype"
    sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    B = sl.shape[0]
    d = qa.shape[-1]
    it = _items(B, h_q, items)
    out = np.zeros((it.shape[0], d), dtype=np.float64)
    rc = lib.oracle_attn(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, _ptr(sl, ctypes.c_int32),
                         B, h_q, h_kv, d, float(scale), dt, _ptr(it, ctypes.c_int32), it.shape[0],
                         nthreads, _ptr(out, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle_attn: bad arguments")
    return out


def _partials(lib, q, k, v, seqlens, h_q: int, h_kv: int, scale: float, n_splits: int = 0,
             chunk_len: int = 0, n_out_splits: int | None = None, items=None, nthreads: int = 0):
    """Per-split (m, l, o) triplets in fp64.

    Exactly one of ``n_splits`` (L_b = ceil(S_b / n_splits)) or ``chunk_len``
    (fixed chunks) selects the split policy.  Returns m, l [n_items, n_out]
    and o [n_items, n_out, d]; an empty split is (-inf, 0, 0)."""
    qa, dt = _raw(q)
    ka, _ = _raw(k)
    va, _ = _raw(v)
    sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    B = sl.shape[0]
    d = qa.shape[-1]
    if n_out_splits is None:
        if n_splits > 0:
            n_out_splits = n_splits
        else:
            n_out_splits = max(1, -(-int(sl.max(initial=0)) // chunk_len))
    it = _items(B, h_q, items)
    n = it.shape[0]
    m = np.zeros((n, n_out_splits), dtype=np.float64)
    l = np.zeros((n, n_out_splits), dtype=np.float64)
    o = np.zeros((n, n_out_splits, d), dtype=np.float64)
    rc = lib.oracle_partials(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, _ptr(sl, ctypes.c_int32),
                             B, h_q, h_kv, d, float(scale), dt, n_splits, chunk_len, n_out_splits,
                             _ptr(it, ctypes.c_int32), n, nthreads,
                             _ptr(m, ctypes.c_double), _ptr(l, ctypes.c_double), _ptr(o, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle_partials: bad arguments")
    return m, l, o


def _merge(lib, m, l, o):
    """Merge triplets with the page's pairwise log-sum-exp rule, then o / l.

    m, l: [rows, n]; o: [rows, n, d] (any float dtype; used as fp64)."""
    m = np.ascontiguousarray(np.asarray(m, dtype=np.float64))
    l = np.ascontiguousarray(np.asarray(l, dtype=np.float64))
    o = np.ascontiguousarray(np.asarray(o, dtype=np.float64))
    rows, n = m.shape
    d = o.shape[-1]
    assert l.shape == (rows, n) and o.shape == (rows, n, d)
    out = np.zeros((rows, d), dtype=np.float64)
    lib.oracle_merge(_ptr(m, ctypes.c_double), _ptr(l, ctypes.c_double), _ptr(o, ctypes.c_double),
                     rows, n, d, _ptr(out, ctypes.c_double))
    return out
