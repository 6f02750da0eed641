"""Sequence-sharded decode, host path on CPU: gloo ranks shard the cache,
exchange packed triplet buffers, and the merge of the gathered triplets
(rank-major) must equal full attention.  The oracle stands in for the
per-rank kernels here (no GPU); the GPU test runs the kernels."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_ranges_cover_each_sequence_once():
    from gqa_split_kv_decode_b200.sharded import shard_range
    for S in [0, 1, 2, 7, 100, 8192, 1 << 20]:
        for world in [1, 2, 3, 8]:
            spans = [shard_range(S, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == S
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c and a <= b
            lens = [b - a for a, b in spans]
            assert max(lens) - min(lens) <= 1
    with pytest.raises(ValueError):
        shard_range(10, 2, 2)


def test_shard_packed_cache_rows():
    from gqa_split_kv_decode_b200.sharded import shard_packed_cache
    sl = torch.tensor([5, 0, 3], dtype=torch.int32)
    k = torch.arange(8, dtype=torch.float32).view(8, 1, 1)
    parts = [shard_packed_cache(k, k, sl, r, 2) for r in range(2)]
    assert parts[0][0].view(-1).tolist() == [0, 1, 5]          # seq 0 keys 0-1, seq 2 key 0
    assert parts[1][0].view(-1).tolist() == [2, 3, 4, 6, 7]    # seq 0 keys 2-4, seq 2 keys 1-2
    assert parts[0][2].tolist() == [2, 0, 1] and parts[1][2].tolist() == [3, 0, 2]


def test_triplet_layout_is_aligned_and_disjoint():
    from gqa_split_kv_decode_b200.sharded import triplet_layout
    for rows, n, d in [(1, 1, 1), (3, 5, 7), (512, 8, 128), (64, 3, 64)]:
        o_off, m_off, l_off, length = triplet_layout(rows, n, d)
        assert o_off == 0 and m_off >= rows * n * d and l_off >= m_off + rows * n
        assert length >= l_off + rows * n
        assert all(x % 4 == 0 for x in (m_off, l_off, length))   # 16-byte segments


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import oracle
    from gqa_split_kv_decode_b200 import sharded
    from workloads import random_case
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        B, hq, hkv, d, n = 3, 8, 2, 64, 3
        w = random_case(B, hq, hkv, d, [37, 0, 200], dtype="f32", seed=5)
        c = w.cfg
        k_loc, v_loc, sl_loc = sharded.shard_packed_cache(w.k, w.v, w.seqlens, rank, world)
        m, l, o = oracle.partials(w.q, k_loc, v_loc, sl_loc, hq, hkv, c.scale, n_splits=n)
        *_, length = sharded.triplet_layout(B * hq, n, d)
        mine = torch.zeros(length, dtype=torch.float64)
        mv, lv, ov = sharded.triplet_views(mine, B, hq, n, d)
        mv.copy_(torch.from_numpy(m).view(B, hq, n))
        lv.copy_(torch.from_numpy(l).view(B, hq, n))
        ov.copy_(torch.from_numpy(o).view(B, hq, n, d))
        gathered = sharded.exchange(mine, world)
        parts = [sharded.triplet_views(gathered[r], B, hq, n, d) for r in range(world)]
        M = torch.cat([p[0].reshape(B * hq, n) for p in parts], dim=1).numpy()   # rank-major
        L = torch.cat([p[1].reshape(B * hq, n) for p in parts], dim=1).numpy()
        O = torch.cat([p[2].reshape(B * hq, n, d) for p in parts], dim=1).numpy()
        got = oracle.merge(M, L, O)
        ref = oracle.attn(w.q, w.k, w.v, w.seqlens, hq, hkv, c.scale)
        q.put((rank, float(np.abs(got - ref).max()), bool(np.isfinite(got).all())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_exchange_and_merge_to_full_attention(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert [g[0] for g in got] == list(range(world))
    for _, err, finite in got:
        assert finite and err < 1e-12
