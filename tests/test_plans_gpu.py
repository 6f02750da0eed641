"""Each launch plan of the fused bf16 path against the oracle.

The plan follows from the grid size (units = splits x kv heads x head blocks
x batch) against R, the per-split CTAs resident at once (2 per SM at d = 128,
4 at d = 64): one wave (units <= R), persistent (R < units <= 4R), many waves
(units > 4R).  One launch merges by ticket inside the kernel; two launches
store the split triplets and merge them in a second kernel (the persistent
plan, and the one-wave plan for groups of 8 or more query heads).  The
shapes below land in each plan on a 148-SM B200.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import random_case

pytestmark = pytest.mark.gpu

TOL = (2e-3, 1e-2)


@pytest.fixture(scope="module")
def gk():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gqa_split_kv_decode_b200 as gk
    return gk


def _check(got, w):
    c = w.cfg
    ref = oracle.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale).reshape(c.B, c.h_q, c.d)
    got = got.double().cpu().numpy()
    err = np.abs(got - ref)
    bound = TOL[0] + TOL[1] * np.abs(ref)
    assert (err <= bound).all(), float((err - bound).max())


# (B, h_q, h_kv, d, seqlens, n_splits, plan and launches expected on 148 SMs)
CASES = [
    (3, 16, 2, 128, [100, 0, 2000], 4, "one_wave", 2),          # merge kernel (G = 8)
    (3, 16, 4, 128, [100, 0, 2000], 4, "one_wave", 1),          # ticket merge (G = 4)
    (4, 64, 8, 128, [0, 1, 17, 3000], 16, "persistent", 2),     # empty and 1-key sequences
    (4, 64, 4, 128, [900, 2, 0, 4000], 32, "persistent", 2),    # 16-head blocks
    (6, 64, 8, 64, [300, 40, 5000, 1, 77, 1200], 16, "persistent", 2),  # d = 64 (R = 4 per SM)
    # the persistent grid takes as few CTAs as cover the slots in the same
    # number of rounds: 768 slots -> 3 rounds of 256 CTAs, 1152 -> 4 of 288,
    # 304 (just past one wave) -> 2 of 152
    (6, 64, 8, 128, [1500, 0, 900, 33, 4096, 2000], 16, "persistent", 2),
    (8, 64, 8, 128, [(733 * i) % 3000 + 1 for i in range(8)], 18, "persistent", 2),
    (1, 64, 8, 128, [9000], 38, "persistent", 2),
    (6, 64, 8, 128, [5, 0, 700, 33, 4096, 16], 32, "many_waves", 1),
    (2, 96, 2, 128, [2500, 300], 200, "many_waves", 1),         # 3 head blocks of 16
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}_hq{c[1]}_hkv{c[2]}_d{c[3]}_n{c[5]}" for c in CASES])
def test_plan_matches_oracle(gk, case):
    B, hq, hkv, d, seqlens, n, plan, launches = case
    w = random_case(B, hq, hkv, d, seqlens, dtype="bf16", seed=sum(seqlens) % 997)
    c = w.cfg
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert gk.fused_plan(B, hq, hkv, d, n) == plan
        assert gk.launches_per_call(B, hq, hkv, d, n) == launches
    assert gk.fused_plan(B, hq, hkv, d, n, dtype=gk.F32) == "simt"
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    for _ in range(2):  # twice: the second call reuses the workspace
        out = gk.gqa_decode_attn(q, k, v, sl, n, c.scale)
        torch.cuda.synchronize()
        assert gk.get_status() == 0
        _check(out, w)


def test_persistent_chunked_ragged(gk):
    """Chunked policy in the persistent plan: 16 sequences, chunk 64."""
    rng = np.random.default_rng(5)
    seqlens = [int(x) for x in rng.integers(0, 300, size=16)]
    seqlens[3] = 0
    w = random_case(16, 32, 8, 128, seqlens, dtype="bf16", seed=6)
    c = w.cfg
    n_slots = -(-max(seqlens) // 64)
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert gk.launches_per_call(16, 32, 8, 128, n_slots) == 2
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    out = gk.gqa_decode_attn_chunked(q, k, v, sl, 64, max(seqlens), c.scale)
    torch.cuda.synchronize()
    assert gk.get_status() == 0
    _check(out, w)


def test_persistent_reports_bad_lengths(gk):
    w = random_case(4, 64, 8, 128, [100, 200, 300, 400], dtype="bf16", seed=7)
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    sl[1] = -3
    out = gk.gqa_decode_attn(q, k, v, sl, 16, w.cfg.scale)
    assert gk.get_status() == gk.ERR_DEVICE_SEQLEN
    assert torch.all(out[1] == 0)
    assert gk.get_status() == 0
    sl[1] = 200
    out = gk.gqa_decode_attn_chunked(q, k, v, sl, 16, 256, w.cfg.scale)  # 400 > 256
    assert gk.get_status() == gk.ERR_DEVICE_SEQLEN


@pytest.mark.parametrize("case", [(8, 64, 8, 128, 8192), (1, 32, 32, 128, 4096), (3, 16, 2, 64, 700)])
def test_auto_split_count(gk, case):
    """n_splits = 0 picks the largest count that fits one wave; the result is
    the oracle's whatever the count."""
    B, hq, hkv, d, S = case
    n = gk.auto_splits(B, hq, hkv, d)
    assert 1 <= n <= 1024
    # one wave: the ticket merge (one launch), or a merge kernel for G >= 8
    assert gk.launches_per_call(B, hq, hkv, d, n) == (2 if hq // hkv >= 8 else 1)
    assert gk.auto_splits(B, hq, hkv, d, max_seqlen=300) <= 2  # >= 256 keys per split
    w = random_case(B, hq, hkv, d, [S] * B if B > 1 else [S], dtype="bf16", seed=B + S)
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    out = gk.gqa_decode_attn(q, k, v, sl, 0, w.cfg.scale)
    torch.cuda.synchronize()
    assert gk.get_status() == 0
    _check(out, w)


@pytest.mark.parametrize("n_splits", [4, 16])   # one wave / persistent plan on a B200
def test_fused_call_replays_in_a_cuda_graph(gk, n_splits):
    """A fused call with an explicit workspace and output captures into a CUDA
    graph (no host synchronisation, no allocation) and replays with new
    inputs copied into the captured buffers."""
    B, hq, hkv, d = 4, 64, 8, 128
    w = random_case(B, hq, hkv, d, [900, 40, 2000, 1], dtype="bf16", seed=31)
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    out = torch.empty(B, hq, d, device="cuda")
    ws = torch.zeros(gk.workspace_size(B, hq, hkv, d, n_splits), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up off the capture
        gk.gqa_decode_attn(q, k, v, sl, n_splits, w.cfg.scale, out=out, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        gk.gqa_decode_attn(q, k, v, sl, n_splits, w.cfg.scale, out=out, workspace=ws)
    for seed in range(3):
        q.copy_(torch.randn(B, hq, d, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16))
        g.replay()
        torch.cuda.synchronize()
        ref = gk.gqa_decode_attn(q, k, v, sl, n_splits, w.cfg.scale)
        assert torch.allclose(out, ref, atol=0, rtol=0)
    assert gk.get_status() == 0
