"""The C-ABI library loads, exports every declared entry point, and rejects
bad arguments on the host (no GPU needed: nothing here launches a kernel)."""
import ctypes
import os
import re

import pytest

import importlib.util

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
HEADERS = sorted(os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h"))

OK, INVALID, UNSUPPORTED, CUDA_ERR, WORKSPACE = 0, 1, 2, 3, 4


def _builder():
    path = os.path.join(ROOT, "gqa_split_kv_decode_b200", "_build.py")
    spec = importlib.util.spec_from_file_location("gqa_decode_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module")
def lib():
    path = _builder().build()
    lib = ctypes.CDLL(path)
    vp, ci, cf, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    ll = ctypes.c_longlong
    lib.gqa_decode_attn.argtypes = [vp, vp, vp, vp, ll, vp, ci, ci, ci, ci, ci, cf, ci, vp, sz, vp]
    lib.gqa_decode_attn_chunked.argtypes = [vp, vp, vp, vp, ll, vp, ci, ci, ci, ci, ci, ci, cf, ci, vp, sz,
                                            vp]
    lib.gqa_decode_partial.argtypes = [vp, vp, vp, vp, ll, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, vp]
    lib.mlo_merge.argtypes = [vp, vp, vp, vp, ci, ci, ci, vp]
    lib.gqa_prefill_attn.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, vp]
    lib.gqa_decode_workspace_size.restype = sz
    lib.gqa_decode_workspace_size.argtypes = [ci] * 5
    lib.gqa_decode_chunked_workspace_size.restype = sz
    lib.gqa_decode_chunked_workspace_size.argtypes = [ci] * 6
    lib.gqa_decode_error_string.restype = ctypes.c_char_p
    return lib


def declared_functions():
    names = []
    for h in HEADERS:
        names += re.findall(r"GQA_API\s+[\w\s\*]+?\b(\w+)\s*\(", open(h).read())
    return names


def test_header_declares_the_path():
    names = set(declared_functions())
    for required in ["gqa_decode_attn", "gqa_decode_partial", "mlo_merge", "gqa_decode_attn_chunked",
                     "gqa_decode_get_status", "gqa_decode_workspace_size", "gqa_prefill_attn"]:
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), f"{n} declared in a header but not exported"


def test_checked_build_exports_the_same_entry_points(lib):
    """libgqadecode_checked.so (index checks on) has every declared entry
    point; each library reports which build it is, and the normal one has no
    checks to test or report."""
    checked = ctypes.CDLL(_builder().build(checked=True))
    for n in declared_functions():
        assert hasattr(checked, n), f"{n} missing from the checked build"
    assert checked.gqa_decode_checked_build() == 1
    assert lib.gqa_decode_checked_build() == 0
    lib.gqa_decode_selftest_bounds.argtypes = [ctypes.c_void_p]
    assert lib.gqa_decode_selftest_bounds(None) == UNSUPPORTED
    lib.gqa_decode_bounds_report.argtypes = [ctypes.c_void_p]
    lib.gqa_decode_bounds_report.restype = ctypes.c_ulonglong
    assert lib.gqa_decode_bounds_report(None) == 0


def test_version_and_error_strings(lib):
    assert lib.gqa_decode_version() >= 100
    for code in range(8):
        assert lib.gqa_decode_error_string(code).startswith(b"GQA_")
    assert b"unknown" in lib.gqa_decode_error_string(99)


FAKE = 0x10000  # aligned, never dereferenced: every call below fails validation first


@pytest.mark.parametrize("kw,expect", [
    (dict(h_q=6, h_kv=4), INVALID),          # h_q not a multiple of h_kv
    (dict(d=96), UNSUPPORTED),               # head dim other than 64 / 128
    (dict(d=0), INVALID),
    (dict(n_splits=-1), INVALID),
    (dict(n_splits=1025), INVALID),
    (dict(scale=float("inf")), INVALID),
    (dict(scale=float("nan")), INVALID),
    (dict(dtype=7), INVALID),
    (dict(B=-1), INVALID),
    (dict(q=0), INVALID),                    # null pointer
    (dict(k=FAKE + 8), INVALID),             # misaligned cache
    (dict(out=FAKE + 4), INVALID),           # misaligned output
    (dict(ws=FAKE, ws_bytes=16), WORKSPACE),  # caller workspace too small
    (dict(ws=FAKE + 16, ws_bytes=1 << 30), WORKSPACE),  # not 256-byte aligned
    (dict(B=0), OK),                         # empty batch: nothing to do
    (dict(B=0, kv_rows=-1), OK),             # cache rows not given
    (dict(kv_rows=-2), INVALID),             # below -1
    (dict(kv_rows=1 << 31), UNSUPPORTED),    # past int32 row coordinates
])
def test_fused_argument_checks(lib, kw, expect):
    a = dict(q=FAKE, k=FAKE, v=FAKE, sl=FAKE, kv_rows=100, out=FAKE, B=1, h_q=8, h_kv=2, d=128,
             n_splits=4, scale=0.1, dtype=1, ws=None, ws_bytes=0)
    a.update(kw)
    rc = lib.gqa_decode_attn(a["q"], a["k"], a["v"], a["sl"], a["kv_rows"], a["out"], a["B"], a["h_q"],
                             a["h_kv"], a["d"], a["n_splits"], a["scale"], a["dtype"], a["ws"],
                             a["ws_bytes"], None)
    assert rc == expect


def test_chunked_argument_checks(lib):
    args = [FAKE] * 4 + [100, FAKE]   # q, k, v, seqlens, kv_rows, out
    assert lib.gqa_decode_attn_chunked(*args, 1, 8, 2, 128, 0, 100, 0.1, 1, None, 0, None) == INVALID
    assert lib.gqa_decode_attn_chunked(*args, 1, 8, 2, 128, 16, -1, 0.1, 1, None, 0, None) == INVALID
    # 1025 chunks of 1 key exceeds the 1024 triplet slots
    assert lib.gqa_decode_attn_chunked(*args, 1, 8, 2, 128, 1, 1025, 0.1, 1, None, 0, None) == INVALID


def test_partial_and_merge_argument_checks(lib):
    p_null = [FAKE] * 4 + [100, 0, FAKE, FAKE]   # q, k, v, seqlens, kv_rows, m = NULL, l, o
    assert lib.gqa_decode_partial(*p_null, 1, 8, 2, 128, 4, 0.1, 1, None) == INVALID
    assert lib.mlo_merge(FAKE, FAKE, FAKE, FAKE, 0, 4, 128, None) == OK     # no rows: no launch
    assert lib.mlo_merge(FAKE, FAKE, FAKE, FAKE, 4, 0, 128, None) == INVALID
    assert lib.mlo_merge(FAKE, FAKE, FAKE, FAKE, 4, 4, 257, None) == INVALID
    assert lib.mlo_merge(0, FAKE, FAKE, FAKE, 4, 4, 128, None) == INVALID


def test_workspace_size_arithmetic(lib):
    """Fixed 256 KiB ticket area, then fp32 triplets: m, l [B*h_q][n] and
    o [B*h_q][n][d], each 256-byte rounded."""
    r = lambda x: (x + 255) // 256 * 256
    T = 256 * 1024

    def expect(B, hq, d, n):
        return T + 2 * r(B * hq * n * 4) + r(B * hq * n * d * 4)

    assert lib.gqa_decode_workspace_size(8, 64, 8, 128, 8) == expect(8, 64, 128, 8)
    assert lib.gqa_decode_workspace_size(1, 32, 1, 128, 2) == expect(1, 32, 128, 2)
    assert lib.gqa_decode_chunked_workspace_size(64, 32, 8, 128, 1024, 32768) == expect(64, 32, 128, 32)
    assert lib.gqa_decode_workspace_size(1, 6, 4, 128, 4) == 0
    assert lib.gqa_decode_workspace_size(1, 8, 2, 96, 4) == 0
    # more than 65536 tickets (B * h_kv * head blocks) is refused
    assert lib.gqa_decode_workspace_size(65535, 8, 2, 128, 1) == 0


def test_launch_count_query_without_a_gpu(lib):
    lib.gqa_decode_launches_per_call.argtypes = [ctypes.c_int] * 6
    assert lib.gqa_decode_launches_per_call(0, 8, 2, 128, 4, 1) == 0      # empty batch
    assert lib.gqa_decode_launches_per_call(2, 8, 2, 128, 4, 0) == 1      # fp32: one kernel
    assert lib.gqa_decode_launches_per_call(2, 6, 4, 128, 4, 1) == -INVALID
    lib.gqa_decode_fused_plan.argtypes = [ctypes.c_int] * 6
    assert lib.gqa_decode_fused_plan(2, 8, 2, 128, 4, 0) == 0          # fp32: the CUDA-core kernel
    assert lib.gqa_decode_fused_plan(2, 6, 4, 128, 4, 1) == -INVALID    # h_q not a multiple of h_kv
    assert lib.gqa_decode_fused_plan(0, 8, 2, 128, 4, 1) == -INVALID    # nothing to plan


@pytest.mark.parametrize("kw,expect", [
    (dict(h_q=6, h_kv=4), INVALID),
    (dict(d=64), UNSUPPORTED),               # prefill runs d_head = 128 only
    (dict(d=0), INVALID),
    (dict(dtype=0), UNSUPPORTED),            # fp32 prefill is not provided
    (dict(dtype=7), INVALID),
    (dict(scale=float("nan")), INVALID),
    (dict(B=-1), INVALID),
    (dict(rows=-1), INVALID),
    (dict(max_seqlen=-1), INVALID),
    (dict(max_seqlen=0), INVALID),           # rows exist, so some sequence is longer
    (dict(max_seqlen=128 * 65536), UNSUPPORTED),
    (dict(q=0), INVALID),
    (dict(v=FAKE + 8), INVALID),             # misaligned
    (dict(out=FAKE + 4), INVALID),
    (dict(B=0), OK),                         # nothing to do
    (dict(rows=0), OK),
])
def test_prefill_argument_checks(lib, kw, expect):
    a = dict(q=FAKE, k=FAKE, v=FAKE, sl=FAKE, out=FAKE, B=2, rows=300, max_seqlen=200, h_q=8, h_kv=2,
             d=128, scale=0.1, dtype=1)
    a.update(kw)
    rc = lib.gqa_prefill_attn(a["q"], a["k"], a["v"], a["sl"], a["out"], a["B"], a["rows"],
                              a["max_seqlen"], a["h_q"], a["h_kv"], a["d"], a["scale"], a["dtype"], None)
    assert rc == expect


def test_ranked_merge_argument_checks(lib):
    ll = ctypes.c_longlong
    lib.mlo_merge_ranked.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 4 + [ll, ll, ctypes.c_void_p]
    ok_args = (FAKE, FAKE, FAKE, FAKE, 4, 2, 3, 128, 4 * 3, 4 * 3 * 128, None)
    assert lib.mlo_merge_ranked(FAKE, FAKE, FAKE, FAKE, 0, 2, 3, 128, 12, 1536, None) == OK   # no rows
    assert lib.mlo_merge_ranked(FAKE, FAKE, FAKE, FAKE, 4, 0, 3, 128, 12, 1536, None) == INVALID
    assert lib.mlo_merge_ranked(FAKE, FAKE, FAKE, FAKE, 4, 2, 3, 257, 12, 1536, None) == INVALID
    assert lib.mlo_merge_ranked(FAKE, FAKE, FAKE, FAKE, 4, 2, 3, 128, 11, 1536, None) == INVALID  # overlap
    assert lib.mlo_merge_ranked(FAKE, FAKE, FAKE, FAKE, 4, 2, 3, 128, 12, 1535, None) == INVALID
    assert lib.mlo_merge_ranked(0, *ok_args[1:]) == INVALID
    assert lib.mlo_merge_ranked(FAKE, FAKE, FAKE, FAKE + 2, *ok_args[4:]) == INVALID           # misaligned
