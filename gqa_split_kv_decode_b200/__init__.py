"""Grouped-query split-KV decode attention for NVIDIA B200 (sm_100a).

Thin ctypes binding over ``libgqadecode.so`` (C ABI in ``include/gqa_decode.h``).
PyTorch is used for device memory and the current stream only: every step of
the computation runs in the library's CUDA kernels.  If the library is
missing, importing this package raises ImportError -- there is no fallback.

Causal prefill (``include/gqa_prefill.h``): ``gqa_prefill_attn`` with q packed
[sum S_b, h_q, d], k, v [sum S_b, h_kv, d], out fp32 [sum S_b, h_q, d].

Decode layouts (see the header): q [B, h_q, d]; k_cache, v_cache packed
[sum S_b, h_kv, d]; seqlens int32 [B] on the device; out fp32 [B, h_q, d];
triplets m, l [B, h_q, n_slots] and o [B, h_q, n_slots, d] in fp32.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "gqa_decode_attn", "gqa_decode_attn_noalloc", "gqa_decode_attn_append", "gqa_decode_attn_chunked", "gqa_decode_partial",
    "gqa_decode_partial_chunked", "mlo_merge", "workspace_size", "chunked_workspace_size",
    "gqa_prefill_attn", "mlo_merge_ranked", "mlo_merge_ranked_raw", "get_status", "auto_splits", "launches_per_call", "fused_plan", "set_wait_timeout_ns", "selftest_wait_timeout", "release", "version",
    "checked_build", "bounds_report", "selftest_bounds",
    "GQADecodeError", "LIB_PATH", "F32", "BF16",
]

# GQA_DECODE_CHECKED=1 loads the checked build (index checks on the kernels'
# derived global accesses; same entry points and results).
_LIB_NAME = "libgqadecode_checked.so" if os.environ.get("GQA_DECODE_CHECKED") == "1" else "libgqadecode.so"
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), _LIB_NAME)
F32, BF16 = 0, 1
(OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE, ERR_DEVICE_TIMEOUT, ERR_DEVICE_SEQLEN,
 ERR_DEVICE_BOUNDS) = range(8)

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python gqa_split_kv_decode_b200/_build.py` "
        "(nvcc, sm_100a). There is no CPU or eager fallback.")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _sz, _ci, _cf, _ull = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float, ctypes.c_ulonglong


def _sig(name, res, *args):
    fn = getattr(_lib, name)
    fn.restype = res
    fn.argtypes = list(args)
    return fn


_version = _sig("gqa_decode_version", _ci)
_errstr = _sig("gqa_decode_error_string", ctypes.c_char_p, _ci)
_ws_size = _sig("gqa_decode_workspace_size", _sz, _ci, _ci, _ci, _ci, _ci)
_ws_size_chunked = _sig("gqa_decode_chunked_workspace_size", _sz, _ci, _ci, _ci, _ci, _ci, _ci)
_ll = ctypes.c_longlong
# packed-cache calls: (q, k_cache, v_cache, seqlens, kv_rows, ...)
_attn = _sig("gqa_decode_attn", _ci, _vp, _vp, _vp, _vp, _ll, _vp, _ci, _ci, _ci, _ci, _ci, _cf,
             _ci, _vp, _sz, _vp)
_attn_noalloc = _sig("gqa_decode_attn_noalloc", _ci, _vp, _vp, _vp, _vp, _ll, _vp, _ci, _ci, _ci,
                     _ci, _ci, _cf, _ci, _vp)
_attn_append = _sig("gqa_decode_attn_append", _ci, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci,
                    _ci, _ci, _ci, _ci, _cf, _ci, _vp, _sz, _vp)
_attn_chunked = _sig("gqa_decode_attn_chunked", _ci, _vp, _vp, _vp, _vp, _ll, _vp, _ci, _ci, _ci,
                     _ci, _ci, _ci, _cf, _ci, _vp, _sz, _vp)
_partial = _sig("gqa_decode_partial", _ci, _vp, _vp, _vp, _vp, _ll, _vp, _vp, _vp, _ci, _ci, _ci,
                _ci, _ci, _cf, _ci, _vp)
_partial_chunked = _sig("gqa_decode_partial_chunked", _ci, _vp, _vp, _vp, _vp, _ll, _vp, _vp, _vp,
                        _ci, _ci, _ci, _ci, _ci, _ci, _cf, _ci, _vp)
_merge = _sig("mlo_merge", _ci, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _vp)
_merge_ranked = _sig("mlo_merge_ranked", _ci, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci,
                     ctypes.c_longlong, ctypes.c_longlong, _vp)
_prefill = _sig("gqa_prefill_attn", _ci, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _cf,
                _ci, _vp)
_get_status = _sig("gqa_decode_get_status", _ci, _vp)
_auto_splits = _sig("gqa_decode_auto_splits", _ci, _ci, _ci, _ci, _ci, _ci)
_launches = _sig("gqa_decode_launches_per_call", _ci, _ci, _ci, _ci, _ci, _ci, _ci)
_plan = _sig("gqa_decode_fused_plan", _ci, _ci, _ci, _ci, _ci, _ci, _ci)
PLAN_NAMES = {0: "simt", 1: "one_wave", 2: "persistent", 3: "many_waves"}
_set_timeout = _sig("gqa_decode_set_wait_timeout_ns", _ci, _ull)
_selftest = _sig("gqa_decode_selftest_wait_timeout", _ci, _ull, _vp)
_release = _sig("gqa_decode_release", _ci)
_checked_build = _sig("gqa_decode_checked_build", _ci)
_bounds_report = _sig("gqa_decode_bounds_report", _ull, _vp)
_selftest_bounds = _sig("gqa_decode_selftest_bounds", _ci, _vp)


class GQADecodeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_errstr(status).decode()}")


def _check(rc: int, where: str):
    if rc != OK:
        raise GQADecodeError(rc, where)


def version() -> int:
    return _version()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"q/k/v must be bf16 or fp32, got {t.dtype}")


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(device) -> int:
    """cudaStream_t of torch's current stream on ``device`` (a torch.device
    or an index)."""
    idx = device if isinstance(device, int) else device.index
    if idx is None:
        idx = torch.cuda.current_device()
    if _raw_stream is not None:
        return _raw_stream(idx)
    return torch.cuda.current_stream(idx).cuda_stream


def _on(idx: int, fn, *args) -> int:
    """Calls the C entry point with device ``idx`` current (switching only
    when another device is)."""
    if torch.cuda.current_device() == idx:
        return fn(*args)
    with torch.cuda.device(idx):
        return fn(*args)


_NAMES = ("q", "k_cache", "v_cache", "seqlens")


def _inputs(q, k_cache, v_cache, seqlens):
    """Checks the decode inputs; returns (B, h_q, h_kv, d, dtype code, device index)."""
    for name, t in zip(_NAMES, (q, k_cache, v_cache, seqlens)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    idx = q.get_device()
    if not (k_cache.get_device() == v_cache.get_device() == seqlens.get_device() == idx):
        raise ValueError("all tensors must be on one device")
    qs, ks = q.shape, k_cache.shape
    if len(qs) != 3 or len(ks) != 3 or v_cache.shape != ks:
        raise ValueError("q must be [B, h_q, d]; k_cache, v_cache [rows, h_kv, d]")
    dt = q.dtype
    if dt != k_cache.dtype or dt != v_cache.dtype:
        raise ValueError("q, k_cache and v_cache must share one dtype")
    if seqlens.dtype != torch.int32 or seqlens.dim() != 1 or seqlens.shape[0] != qs[0]:
        raise ValueError("seqlens must be int32 [B]")
    if qs[2] != ks[2]:
        raise ValueError("head dims differ")
    if dt == torch.bfloat16:
        code = BF16
    elif dt == torch.float32:
        code = F32
    else:
        raise TypeError(f"q/k/v must be bf16 or fp32, got {dt}")
    return qs[0], qs[1], ks[1], qs[2], code, idx


_dummies: dict = {}


def _ptr(t: torch.Tensor) -> int:
    """Device address of a tensor; an empty tensor (a cache with no rows)
    gets a small zeroed placeholder, which the kernels never read because
    every sequence of such a batch has length 0."""
    if t.numel() > 0:
        return t.data_ptr()
    key = (t.device.type, t.device.index)
    if key not in _dummies:
        _dummies[key] = torch.zeros(256, dtype=torch.uint8, device=t.device)
    return _dummies[key].data_ptr()


def _default_scale(d: int, scale):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


_workspaces: dict = {}


def _workspace(device: torch.device, nbytes: int) -> torch.Tensor:
    """Grow-only zero-filled workspace per device, owned by torch's allocator."""
    key = (device.type, device.index)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def _out(out, shape, device):
    if out is None:
        return torch.empty(shape, dtype=torch.float32, device=device)
    if out.dtype != torch.float32 or tuple(out.shape) != tuple(shape) or not out.is_contiguous():
        raise ValueError(f"out must be contiguous fp32 {tuple(shape)}")
    if out.device != device:
        raise ValueError("out must be on the inputs' device")
    return out


def _out_idx(out, shape, idx: int):
    """_out for the decode entry points (device given as an index)."""
    if out is None:
        return torch.empty(shape, dtype=torch.float32, device=torch.device("cuda", idx))
    if (out.dtype != torch.float32 or out.shape != shape or not out.is_contiguous()
            or out.get_device() != idx):
        raise ValueError(f"out must be contiguous fp32 {tuple(shape)} on the inputs' device")
    return out


def _ws(workspace, idx: int, need_fn, *shape):
    """(pointer, bytes) of the caller's workspace, or of the binding's own
    grow-only one sized by need_fn(*shape)."""
    if workspace is None:
        workspace = _workspace(torch.device("cuda", idx), need_fn(*shape))
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def workspace_size(B, h_q, h_kv, d, n_splits) -> int:
    return _ws_size(B, h_q, h_kv, d, n_splits)


def chunked_workspace_size(B, h_q, h_kv, d, chunk_len, max_seqlen) -> int:
    return _ws_size_chunked(B, h_q, h_kv, d, chunk_len, max_seqlen)


def gqa_decode_attn(q, k_cache, v_cache, seqlens, n_splits: int, scale=None, out=None,
                    workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Fused split-KV decode attention (split by count); returns fp32 [B, h_q, d]."""
    B, h_q, h_kv, d, dt, idx = _inputs(q, k_cache, v_cache, seqlens)
    out = _out_idx(out, (B, h_q, d), idx)
    wp, wb = _ws(workspace, idx, _ws_size, B, h_q, h_kv, d, n_splits)
    _check(_on(idx, _attn, q.data_ptr(), _ptr(k_cache), _ptr(v_cache), seqlens.data_ptr(),
               k_cache.shape[0], out.data_ptr(), B, h_q, h_kv, d, n_splits, _default_scale(d, scale), dt, wp, wb,
               _stream(idx)), "gqa_decode_attn")
    return out


def gqa_decode_attn_noalloc(q, k_cache, v_cache, seqlens, n_splits: int, scale=None,
                            out=None) -> torch.Tensor:
    """gqa_decode_attn for callers that cannot allocate device memory.

    The scratch is a fixed 40 MiB array inside the library (one per device),
    so the call itself allocates nothing; shapes that need more scratch raise
    GQADecodeError (ERR_WORKSPACE).  Calls share that array: keep them on one
    stream.  (Passing ``out=None`` still lets torch allocate the result here;
    pass ``out`` to avoid even that.)"""
    B, h_q, h_kv, d, dt, idx = _inputs(q, k_cache, v_cache, seqlens)
    out = _out_idx(out, (B, h_q, d), idx)
    _check(_on(idx, _attn_noalloc, q.data_ptr(), _ptr(k_cache), _ptr(v_cache), seqlens.data_ptr(),
               k_cache.shape[0], out.data_ptr(), B, h_q, h_kv, d, n_splits, _default_scale(d, scale), dt,
               _stream(idx)), "gqa_decode_attn_noalloc")
    return out


def gqa_decode_attn_append(q, k_new, v_new, k_cache, v_cache, seqlens, n_splits: int, scale=None,
                           out=None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Writes k_new, v_new ([B, h_kv, d]) into the padded cache ([B, cap, h_kv, d])
    at row seqlens[b] of each sequence and attends over the seqlens[b] + 1
    keys.  seqlens is left unchanged (advance it for the next step)."""
    if k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache, v_cache must be [B, cap, h_kv, d]")
    B, cap, h_kv, d = k_cache.shape
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        if not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (B, h_kv, d) or t.dtype != q.dtype:
            raise ValueError(f"{name} must be a contiguous CUDA tensor [B, h_kv, d] of q's dtype")
        if t.get_device() != q.get_device():
            raise ValueError(f"{name} must be on q's device")
    _, h_q, _, _, dt, idx = _inputs(q, k_cache.view(B * cap, h_kv, d), v_cache.view(B * cap, h_kv, d),
                                    seqlens)
    out = _out_idx(out, (B, h_q, d), idx)
    wp, wb = _ws(workspace, idx, _ws_size, B, h_q, h_kv, d, n_splits)
    _check(_on(idx, _attn_append, q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), k_cache.data_ptr(),
               v_cache.data_ptr(), seqlens.data_ptr(), out.data_ptr(), B, h_q, h_kv, d, cap, n_splits,
               _default_scale(d, scale), dt, wp, wb, _stream(idx)), "gqa_decode_attn_append")
    return out


def gqa_decode_attn_chunked(q, k_cache, v_cache, seqlens, chunk_len: int, max_seqlen: int,
                            scale=None, out=None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Fused split-KV decode attention with fixed chunks (ragged batches)."""
    B, h_q, h_kv, d, dt, idx = _inputs(q, k_cache, v_cache, seqlens)
    out = _out_idx(out, (B, h_q, d), idx)
    wp, wb = _ws(workspace, idx, _ws_size_chunked, B, h_q, h_kv, d, chunk_len, max_seqlen)
    _check(_on(idx, _attn_chunked, q.data_ptr(), _ptr(k_cache), _ptr(v_cache), seqlens.data_ptr(),
               k_cache.shape[0], out.data_ptr(), B, h_q, h_kv, d, chunk_len, max_seqlen, _default_scale(d, scale), dt,
               wp, wb, _stream(idx)), "gqa_decode_attn_chunked")
    return out


def _triplets(B, h_q, n, d, idx, m, l, o):
    m = _out_idx(m, (B, h_q, n), idx)
    l = _out_idx(l, (B, h_q, n), idx)
    o = _out_idx(o, (B, h_q, n, d), idx)
    return m, l, o


def gqa_decode_partial(q, k_cache, v_cache, seqlens, n_splits: int, scale=None, m=None, l=None, o=None):
    """Per-split (m, l, o) triplets (split by count)."""
    B, h_q, h_kv, d, dt, idx = _inputs(q, k_cache, v_cache, seqlens)
    m, l, o = _triplets(B, h_q, n_splits, d, idx, m, l, o)
    _check(_on(idx, _partial, q.data_ptr(), _ptr(k_cache), _ptr(v_cache), seqlens.data_ptr(),
               k_cache.shape[0], m.data_ptr(), l.data_ptr(), o.data_ptr(), B, h_q, h_kv, d, n_splits,
               _default_scale(d, scale), dt, _stream(idx)), "gqa_decode_partial")
    return m, l, o


def gqa_decode_partial_chunked(q, k_cache, v_cache, seqlens, chunk_len: int, max_seqlen: int,
                               scale=None, m=None, l=None, o=None):
    """Per-chunk (m, l, o) triplets; n_slots = max(1, ceil(max_seqlen / chunk_len))."""
    B, h_q, h_kv, d, dt, idx = _inputs(q, k_cache, v_cache, seqlens)
    n = max(1, -(-max_seqlen // chunk_len)) if chunk_len > 0 and max_seqlen >= 0 else 1
    m, l, o = _triplets(B, h_q, n, d, idx, m, l, o)
    _check(_on(idx, _partial_chunked, q.data_ptr(), _ptr(k_cache), _ptr(v_cache), seqlens.data_ptr(),
               k_cache.shape[0], m.data_ptr(), l.data_ptr(), o.data_ptr(), B, h_q, h_kv, d, chunk_len, max_seqlen,
               _default_scale(d, scale), dt, _stream(idx)), "gqa_decode_partial_chunked")
    return m, l, o


def mlo_merge(m, l, o, out=None) -> torch.Tensor:
    """Log-sum-exp merge + normalisation of [..., n] triplets -> fp32 [..., d]."""
    for name, t in (("m", m), ("l", l), ("o", o)):
        if not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor")
    idx = m.get_device()
    if l.get_device() != idx or o.get_device() != idx:
        raise ValueError("m, l and o must be on one device")
    n, d = o.shape[-2], o.shape[-1]
    lead = tuple(m.shape[:-1])
    if tuple(m.shape) != lead + (n,) or tuple(l.shape) != lead + (n,) or tuple(o.shape) != lead + (n, d):
        raise ValueError("shapes: m, l [..., n]; o [..., n, d]")
    rows = int(math.prod(lead))
    out = _out_idx(out, torch.Size(lead + (d,)), idx)
    _check(_on(idx, _merge, m.data_ptr(), l.data_ptr(), o.data_ptr(), out.data_ptr(), rows, n, d,
               _stream(idx)), "mlo_merge")
    return out


def mlo_merge_ranked(m, l, o, out=None) -> torch.Tensor:
    """Merge of triplets gathered from R shards: m, l [R, ..., n], o
    [R, ..., n, d] -> fp32 [..., d]; a row's splits in rank-major order."""
    for name, t in (("m", m), ("l", l), ("o", o)):
        if not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor")
    R, n, d = m.shape[0], o.shape[-2], o.shape[-1]
    lead = tuple(m.shape[1:-1])
    if (tuple(m.shape) != (R,) + lead + (n,) or tuple(l.shape) != tuple(m.shape)
            or tuple(o.shape) != (R,) + lead + (n, d)):
        raise ValueError("shapes: m, l [R, ..., n]; o [R, ..., n, d]")
    rows = int(math.prod(lead))
    out = _out(out, lead + (d,), m.device)
    return mlo_merge_ranked_raw(m, l, o, out, rows, R, n, d, rows * n, rows * n * d)


def mlo_merge_ranked_raw(m, l, o, out, rows, n_ranks, n_splits, d, stride_ml, stride_o):
    """mlo_merge_ranked on raw views: rank r's m / l block starts r * stride_ml
    elements after ``m`` / ``l``, its o block r * stride_o after ``o`` (the
    tensors only supply device addresses)."""
    with torch.cuda.device(out.device):
        _check(_merge_ranked(m.data_ptr(), l.data_ptr(), o.data_ptr(), out.data_ptr(), rows, n_ranks,
                             n_splits, d, stride_ml, stride_o, _stream(out.device)), "mlo_merge_ranked")
    return out


def auto_splits(B, h_q, h_kv, d, max_seqlen=0, device=None) -> int:
    """Split count a fused call with n_splits=0 uses on ``device`` (largest
    count that fills one wave; >= 256 keys per split when max_seqlen > 0)."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(device):
        n = _auto_splits(B, h_q, h_kv, d, max_seqlen)
    if n < 0:
        raise GQADecodeError(-n, "gqa_decode_auto_splits")
    return n


def launches_per_call(B, h_q, h_kv, d, n_slots, dtype=BF16, device=None) -> int:
    """Kernels one fused call launches for this shape on ``device``."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(device):
        n = _launches(B, h_q, h_kv, d, n_slots, dtype)
    if n < 0:
        raise GQADecodeError(-n, "gqa_decode_launches_per_call")
    return n


def fused_plan(B, h_q, h_kv, d, n_slots, dtype=BF16, device=None) -> str:
    """Launch plan of a fused call for this shape on ``device``: "simt" (fp32),
    "one_wave", "persistent" or "many_waves"."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(device):
        n = _plan(B, h_q, h_kv, d, n_slots, dtype)
    if n < 0:
        raise GQADecodeError(-n, "gqa_decode_fused_plan")
    return PLAN_NAMES[n]


def get_status(device=None) -> int:
    """Synchronise the current stream, read and clear the device status word."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(device):
        return _get_status(_stream(device))


def set_wait_timeout_ns(ns: int) -> None:
    _check(_set_timeout(ns), "gqa_decode_set_wait_timeout_ns")


def selftest_wait_timeout(ns: int, device=None) -> None:
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(device):
        _check(_selftest(ns, _stream(device)), "gqa_decode_selftest_wait_timeout")


def release() -> None:
    _check(_release(), "gqa_decode_release")


def checked_build() -> bool:
    """True when the loaded library is the checked build (GQA_DECODE_CHECKED=1)."""
    return _checked_build() == 1


def bounds_report(device=None):
    """The first failed index check since the last report, as (site, index),
    or None (always None in the normal build).  Synchronises the stream."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(device):
        rec = _bounds_report(_stream(device))
    if rec == 0:
        return None
    if rec == (1 << 64) - 1:
        raise GQADecodeError(ERR_CUDA, "gqa_decode_bounds_report")
    rec -= 1
    return rec >> 56, rec & ((1 << 56) - 1)


def selftest_bounds(device=None) -> None:
    """Checked build: one deliberately failing index check (its store skipped)."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(device):
        _check(_selftest_bounds(_stream(device)), "gqa_decode_selftest_bounds")


def gqa_prefill_attn(q, k, v, seqlens, scale=None, max_seqlen=None, out=None):
    """Causal prefill attention: query i of sequence b attends keys 0..i of
    that sequence.  q [rows, h_q, 128], k, v [rows, h_kv, 128] bf16, packed by
    sequence (rows = sum S_b); seqlens int32 [B] on the device.  Returns fp32
    [rows, h_q, 128].  ``max_seqlen`` bounds every S_b; when omitted it is read
    from ``seqlens`` (one device-to-host copy)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("seqlens", seqlens)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not (q.device == k.device == v.device == seqlens.device):
        raise ValueError("all tensors must be on one device")
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape or q.shape[0] != k.shape[0]:
        raise ValueError("q must be [rows, h_q, d]; k, v [rows, h_kv, d] with the same rows")
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise ValueError("q, k and v must share one dtype")
    if seqlens.dtype != torch.int32 or seqlens.dim() != 1:
        raise ValueError("seqlens must be int32 [B]")
    if q.shape[2] != k.shape[2]:
        raise ValueError("head dims differ")
    rows, h_q, d = q.shape
    B = seqlens.shape[0]
    if max_seqlen is None:
        max_seqlen = int(seqlens.max().item()) if B > 0 else 0
    if out is None:
        out = torch.empty((rows, h_q, d), dtype=torch.float32, device=q.device)
    elif out.shape != (rows, h_q, d) or out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be contiguous fp32 [rows, h_q, d]")
    _check(_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(seqlens), _ptr(out), B, rows, int(max_seqlen),
                    h_q, k.shape[1], d, _default_scale(d, scale), _dtype_code(q),
                    _stream(q.device)), "gqa_prefill_attn")
    return out
