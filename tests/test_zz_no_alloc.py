"""The allocation-free entry point, gqa_decode_attn_noalloc.

It serves callers that cannot call cudaMalloc (a plugin whose host program
owns every device allocation through its own pool, or a latency-critical
path that cannot take cudaMalloc's device-wide synchronisation): its scratch
is a fixed array inside the library instead of a workspace.  These tests
call it through the C ABI (via the ctypes binding) and check it against the
fp64 oracle and against the workspace entry point, gqa_decode_attn, on two
calls in a row -- the second call finds the array as the first one left it.
The shapes cover both kinds of fused plan: the single-launch plans that
merge through tickets in the array, and the two-launch plans (persistent,
or one wave of groups of 8 query heads) whose kernels keep their triplets
there.  This file is collected last so that a
run stopping at the first failure has run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
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
    got = np.asarray(got.double().cpu().numpy() if isinstance(got, torch.Tensor) else got, np.float64)
    ref = np.asarray(ref.double().cpu().numpy() if isinstance(ref, torch.Tensor) else ref, np.float64)
    err = np.abs(got - ref)
    assert (err <= atol + rtol * np.abs(ref)).all(), float((err - atol - rtol * np.abs(ref)).max())


def _oracle(w):
    c = w.cfg
    return oracle.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale).reshape(c.B, c.h_q, c.d)


# (B, h_q, h_kv, d, seqlens, n_splits, dtype, launches per call on a 148-SM B200)
CASES = [
    (3, 32, 8, 128, [3000, 17, 900], 8, "bf16", 1),          # one wave, ticket merge (G = 4)
    (3, 64, 8, 128, [3000, 17, 900], 8, "bf16", 2),          # one wave, merge kernel (G = 8)
    (3, 64, 8, 128, [3000, 17, 900], 8, "f32", 1),
    (4, 64, 8, 128, [0, 1, 17, 3000], 16, "bf16", 2),        # persistent kernel + row merge
    (6, 64, 8, 128, [5, 0, 700, 33, 4096, 16], 32, "bf16", 1),  # many waves, ticket merge
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}_n{c[5]}_{c[6]}_l{c[7]}" for c in CASES])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(gk, case):
    B, hq, hkv, d, seqlens, n, dtype, launches = case
    w = random_case(B, hq, hkv, d, seqlens, dtype=dtype, seed=77 + n)
    c = w.cfg
    if dtype == "bf16" and torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert gk.launches_per_call(B, hq, hkv, d, n) == launches
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    ref = _oracle(w)
    with_ws = gk.gqa_decode_attn(q, k, v, sl, n, c.scale)
    torch.cuda.synchronize()
    assert gk.get_status() == 0
    for _ in range(2):
        got = gk.gqa_decode_attn_noalloc(q, k, v, sl, n, c.scale)
        torch.cuda.synchronize()
        assert gk.get_status() == 0
        _close(got, ref, dtype)
        _close(got, with_ws, dtype)


def test_noalloc_other_shape_after_first(gk):
    """A second shape after the first: tickets of the earlier call do not leak."""
    w = random_case(2, 16, 2, 64, [700, 5], dtype="bf16", seed=78)
    c = w.cfg
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    ref = _oracle(w)
    for _ in range(2):
        got = gk.gqa_decode_attn_noalloc(q, k, v, sl, 4, c.scale)
        torch.cuda.synchronize()
        assert gk.get_status() == 0
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
