"""The allocation-free entry point, gqa_decode_attn_noalloc.

It serves callers that cannot call cudaMalloc (a plugin whose host program
owns every device allocation through its own pool, or a latency-critical
path that cannot take cudaMalloc's device-wide synchronisation): its scratch
is a fixed array inside the library instead of a workspace.  These tests
call it through the C ABI (via the ctypes binding) and check it against the
workspace entry point, gqa_decode_attn, on two calls in a row -- the second
call finds the array as the first one left it.  This file is collected last
so that a run stopping at the first failure has run every other test.
"""
import numpy as np
import pytest
import torch

from workloads import random_case

pytestmark = pytest.mark.gpu

TOL = {"bf16": (2e-3, 1e-2), "f32": (1e-5, 1e-5)}


@pytest.fixture(scope="module")
def gk():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gqa_split_kv_decode_b200 as gk
    return gk


def _close(got, ref, dtype):
    atol, rtol = TOL[dtype]
    got = got.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    err = np.abs(got - ref)
    assert (err <= atol + rtol * np.abs(ref)).all(), float((err - atol - rtol * np.abs(ref)).max())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_workspace_entry_point_twice(gk, dtype):
    w = random_case(3, 64, 8, 128, [3000, 17, 900], dtype=dtype, seed=77)
    c = w.cfg
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    ref = gk.gqa_decode_attn(q, k, v, sl, 8, c.scale)
    for _ in range(2):
        got = gk.gqa_decode_attn_noalloc(q, k, v, sl, 8, c.scale)
        torch.cuda.synchronize()
        assert gk.get_status() == 0
        _close(got, ref, dtype)


def test_noalloc_other_shape_after_first(gk):
    """A second shape after the first: tickets of the earlier call do not leak."""
    w = random_case(2, 16, 2, 64, [700, 5], dtype="bf16", seed=78)
    c = w.cfg
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    ref = gk.gqa_decode_attn(q, k, v, sl, 4, c.scale)
    for _ in range(2):
        got = gk.gqa_decode_attn_noalloc(q, k, v, sl, 4, c.scale)
        _close(got, ref, "bf16")


def test_noalloc_rejects_scratch_beyond_its_limit(gk):
    """A shape whose scratch exceeds the fixed 40 MiB is refused before any
    launch (64 sequences x 64 heads x 64 splits of fp32 triplets ~ 136 MB)."""
    B, hq, hkv, d = 64, 64, 8, 128
    assert gk.workspace_size(B, hq, hkv, d, 64) > 40 << 20
    q = torch.zeros(B, hq, d, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(16, hkv, d, dtype=torch.bfloat16, device="cuda")
    sl = torch.zeros(B, dtype=torch.int32, device="cuda")
    with pytest.raises(gk.GQADecodeError) as e:
        gk.gqa_decode_attn_noalloc(q, kv, kv, sl, 64)
    assert e.value.status == gk.ERR_WORKSPACE
