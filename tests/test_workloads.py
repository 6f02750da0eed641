"""The seeded input recipe (host only): every 2^24-value chunk of q, k and v
is drawn from its own PCG64(SeedSequence([seed, tensor, chunk])), so the
inputs do not depend on how many threads draw them; lengths, bias positions
and the x10 V rows come from PCG64(seed)."""
import numpy as np
import torch

import workloads
from workloads import CHUNK, CONFIGS, random_case, scaled


def _chunk(seed, tensor_id, c, n, std=1.0):
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id, c])))
    x = g.standard_normal(n, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def test_small_case_matches_the_recipe():
    w = random_case(3, 8, 2, 64, [5, 0, 11], dtype="f32", seed=17)
    q = _chunk(17, 0, 0, 3 * 8 * 64)
    k = _chunk(17, 1, 0, 16 * 2 * 64)
    v = _chunk(17, 2, 0, 16 * 2 * 64)
    assert np.array_equal(w.q.numpy().ravel(), q)
    assert np.array_equal(w.k.numpy().ravel(), k)
    assert np.array_equal(w.v.numpy().ravel(), v)


def test_multi_chunk_tensor_matches_the_recipe_and_repeats():
    # 2^24 + 2^20 values of k: two chunks, the second one partial
    rows = (CHUNK + (1 << 20)) // 128
    w = random_case(1, 1, 1, 128, [rows], dtype="bf16", seed=5)
    k = w.k.float().numpy().ravel()
    first = torch.from_numpy(_chunk(5, 1, 0, CHUNK)).to(torch.bfloat16).float().numpy()
    second = torch.from_numpy(_chunk(5, 1, 1, 1 << 20)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(k[:CHUNK], first)
    assert np.array_equal(k[CHUNK:], second)
    again = random_case(1, 1, 1, 128, [rows], dtype="bf16", seed=5)
    assert torch.equal(again.k, w.k) and torch.equal(again.v, w.v)


def test_structures_of_the_workloads():
    # ragged: lengths uniform in [S_min, S] from the main generator
    cfg = scaled("ragged", B=40, S=3000)
    w = workloads.generate(cfg)
    rng = np.random.Generator(np.random.PCG64(cfg.seed))
    want = rng.integers(cfg.S_min, cfg.S, size=cfg.B, endpoint=True)
    assert np.array_equal(w.seqlens.numpy(), want.astype(np.int32))
    # some v rows are x10 (about 1%), the rest standard normal rounded to bf16
    big = (w.v.float().abs().amax(dim=-1) > 6.0).float().mean().item()
    assert 0.003 < big < 0.03
    # llama70b: the +6 logit bias on round(0.001 S) positions per sequence
    c70 = scaled("llama70b", B=2, S=4000)
    w70 = workloads.generate(c70)
    q = w70.q.double()
    k = w70.k.double()
    for b in range(2):
        kb = k[b * 4000:(b + 1) * 4000]
        s = torch.einsum("hd,jd->hj", q[b, :8], kb[:, 0]) * c70.scale   # kv head 0, its 8 query heads
        # the group's mean logit is ~N(0, 1/8) at a plain key and ~6 at a biased one
        high = (s.mean(dim=0) > 3.0).nonzero().numel()
        assert high == round(0.001 * 4000)
    assert CONFIGS["llama70b"].bias_frac == 0.001
