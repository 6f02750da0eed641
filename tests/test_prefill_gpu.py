"""Causal prefill (gqa_prefill_attn, tcgen05 kernel) against the oracle.

Every output of the small cases and of the two full-size workloads is
compared element by element; the 32k-token prompt is compared on sampled
(sequence, head, position) rows that include each 128-row tile's first and
last rows and each sequence's first and last positions.  Bound:
|e| <= 2e-3 + 1e-2 |ref| (bf16 inputs).
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import generate_prefill, prefill_case

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2


@pytest.fixture(scope="module")
def gk():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gqa_split_kv_decode_b200 as gk
    return gk


def _run(gk, w, max_seqlen=None):
    out = gk.gqa_prefill_attn(w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda(), w.scale,
                              max_seqlen=max_seqlen)
    torch.cuda.synchronize()
    return out.cpu().double().numpy()


def _assert_close(got, ref):
    assert np.isfinite(got).all()
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), (int(bad.sum()), float((err - ATOL - RTOL * np.abs(ref)).max()))


def _check_all(gk, w):
    got = _run(gk, w)
    assert gk.get_status() == 0
    ref = oracle.prefill(w.q, w.k, w.v, w.seqlens, w.h_q, w.h_kv, w.scale)
    _assert_close(got.reshape(-1, w.d), ref)


CASES = [
    # seqlens, h_q, h_kv, seed
    ([128], 8, 2, 1),                          # one query tile
    ([300], 8, 8, 2),                          # three tiles, ragged tail, MHA
    ([1, 127, 128, 129, 0, 700, 5], 16, 2, 3),  # ragged batch, an empty sequence
    ([513, 256], 64, 8, 4),                    # Llama-70B head shape
    ([1000], 4, 1, 5),                         # one kv head for all
    ([64, 65, 63, 191, 192, 193], 8, 4, 6),    # lengths around the 64-key tile edges
    ([1] * 5 + [0] * 3 + [2, 3, 40, 17], 4, 4, 7),   # many very short prompts, empty ones between
    ([129], 1, 1, 8),                          # one head
    ([200, 130], 32, 2, 9),                    # group of 16 query heads per kv head
    ([257], 32, 1, 10),                        # group of 32: every head reads one kv head
    ([2047, 1, 2049], 8, 2, 11),               # lengths either side of a 2048 boundary
]


@pytest.mark.parametrize("case", CASES, ids=[f"S{'-'.join(map(str, c[0]))}_hq{c[1]}_hkv{c[2]}" for c in CASES])
def test_prefill_matches_oracle(gk, case):
    seqlens, hq, hkv, seed = case
    _check_all(gk, prefill_case(seqlens, hq, hkv, 128, seed=seed))


@pytest.mark.parametrize("scale", [0.0, -0.05, 0.3])
def test_prefill_scales(gk, scale):
    """scale 0 (every row the running mean of V), a negative scale (the row
    minimum leads), a large scale (sharp softmax)."""
    _check_all(gk, prefill_case([200, 77], 8, 2, 128, seed=11, scale=scale))


def test_prefill_growing_logits_rescale(gk):
    """Logits that grow by ~4.5 (natural log) per 64-key tile along the
    sequence, so the row max keeps rising past the lazy-rescale threshold."""
    w = prefill_case([700], 8, 2, 128, seed=12)
    j = torch.arange(700, dtype=torch.float32)
    k = w.k.float()
    k[:, :, 0] += 0.1 * j[:, None]
    q = w.q.float()
    q[:, :, 0] = 8.0
    w.k, w.q = k.to(torch.bfloat16), q.to(torch.bfloat16)
    _check_all(gk, w)


def test_prefill_falling_logits(gk):
    """The first keys dominate: the reference max is set by tile 0 and never
    moves."""
    w = prefill_case([600], 8, 2, 128, seed=13)
    j = torch.arange(600, dtype=torch.float32)
    k = w.k.float()
    k[:, :, 0] -= 0.1 * j[:, None]
    q = w.q.float()
    q[:, :, 0] = 8.0
    w.k, w.q = k.to(torch.bfloat16), q.to(torch.bfloat16)
    _check_all(gk, w)


def _sample_items(seqlens, h_q, n, seed):
    rng = np.random.default_rng(seed)
    items = set()
    for b, S in enumerate(seqlens):
        for i in {0, S - 1} | {t * 128 for t in range(0, S, 128) if t * 128 < S} | \
                 {min(S - 1, t * 128 + 127) for t in range(0, (S + 127) // 128)}:
            if 0 <= i < S:
                items.add((b, int(rng.integers(h_q)), i))
    nz = [b for b, S in enumerate(seqlens) if S > 0]
    while len(items) < n:
        b = int(rng.choice(nz))
        items.add((b, int(rng.integers(h_q)), int(rng.integers(seqlens[b]))))
    return sorted(items)


@pytest.mark.parametrize("name", ["llama70b_prefill2k", "prefill_ragged"])
def test_prefill_full_size_every_row(gk, name):
    """The two prefill workloads at full size, every output element against
    the oracle (a full fp64 pass takes seconds on the host's cores)."""
    w = generate_prefill(name)
    got = _run(gk, w)
    assert gk.get_status() == 0
    ref = oracle.prefill(w.q, w.k, w.v, w.seqlens, w.h_q, w.h_kv, w.scale)
    _assert_close(got.reshape(-1, w.d), ref)


def test_prefill_long_prompt_sampled(gk):
    """A 32k-token prompt (256 query tiles, the longest first in the grid)
    and a short one beside it: sampled rows against the oracle."""
    w = prefill_case([32768, 200], 4, 1, 128, seed=23)
    got = _run(gk, w)
    assert gk.get_status() == 0
    sl = w.seqlens.tolist()
    items = _sample_items(sl, w.h_q, 700, seed=8)
    ref = oracle.prefill(w.q, w.k, w.v, w.seqlens, w.h_q, w.h_kv, w.scale, items=items)
    off = np.concatenate([[0], np.cumsum(sl)])
    rows = np.array([(off[b] + i) for b, h, i in items])
    heads = np.array([h for b, h, i in items])
    _assert_close(got[rows, heads], ref)


def test_prefill_reports_sequence_over_max(gk):
    """S_b above max_seqlen: the status word says so; the rows inside the
    grid are still right."""
    w = prefill_case([400, 100], 8, 2, 128, seed=14)
    got = _run(gk, w, max_seqlen=256)
    assert gk.get_status() == gk.ERR_DEVICE_SEQLEN
    assert gk.get_status() == 0
    ref = oracle.prefill(w.q, w.k, w.v, w.seqlens, w.h_q, w.h_kv, w.scale).reshape(-1, 8, 128)
    keep = np.r_[0:256, 400:500]
    _assert_close(got[keep], ref[keep])


def test_prefill_back_to_back_calls_agree(gk):
    """Two launches in a row on one stream (the second may start early under
    programmatic dependent launch) give bit-identical results."""
    w = prefill_case([900, 33], 16, 2, 128, seed=15)
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    a = gk.gqa_prefill_attn(q, k, v, sl, w.scale, max_seqlen=900)
    b = gk.gqa_prefill_attn(q, k, v, sl, w.scale, max_seqlen=900)
    torch.cuda.synchronize()
    assert gk.get_status() == 0
    assert torch.equal(a, b)


def test_prefill_rejects_unsupported(gk):
    w = prefill_case([10], 4, 2, 64, seed=16)
    with pytest.raises(gk.GQADecodeError):
        gk.gqa_prefill_attn(w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda())
    w = prefill_case([10], 4, 2, 128, dtype="f32", seed=16)
    with pytest.raises(gk.GQADecodeError):
        gk.gqa_prefill_attn(w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda())


def test_prefill_replays_in_a_cuda_graph(gk):
    """One launch, no host synchronisation and no allocation when max_seqlen
    and out are given: the call captures into a CUDA graph, and a replay on
    new inputs equals a direct call bit for bit."""
    w1 = prefill_case([700, 300], 16, 2, 128, seed=21)
    w2 = prefill_case([700, 300], 16, 2, 128, seed=22)
    q, k, v = w1.q.cuda(), w1.k.cuda(), w1.v.cuda()
    sl = w1.seqlens.cuda()
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        gk.gqa_prefill_attn(q, k, v, sl, w1.scale, max_seqlen=700, out=out)   # warm-up
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        gk.gqa_prefill_attn(q, k, v, sl, w1.scale, max_seqlen=700, out=out)
    q.copy_(w2.q.cuda()); k.copy_(w2.k.cuda()); v.copy_(w2.v.cuda())
    g.replay()
    torch.cuda.synchronize()
    direct = gk.gqa_prefill_attn(w2.q.cuda(), w2.k.cuda(), w2.v.cuda(), sl, w2.scale, max_seqlen=700)
    torch.cuda.synchronize()
    assert gk.get_status() == 0
    assert torch.equal(out, direct)
