"""Sequence-sharded decode on one GPU: the ranks' shards are emulated in one
process (each shard's partial triplets written into its slot of the gathered
buffer, as the all-gather would leave them), then merged by
mlo_merge_ranked.  No rank waits on another, so nothing here needs more
than one GPU."""
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


def _gathered(gk, w, world, n):
    from gqa_split_kv_decode_b200 import sharded
    c = w.cfg
    q = w.q.cuda()
    *_, length = sharded.triplet_layout(c.B * c.h_q, n, c.d)
    gathered = torch.full((world, length), float("nan"), dtype=torch.float32, device="cuda")
    for r in range(world):
        k_loc, v_loc, sl_loc = sharded.shard_packed_cache(w.k, w.v, w.seqlens, r, world)
        m, l, o = sharded.triplet_views(gathered[r], c.B, c.h_q, n, c.d)
        gk.gqa_decode_partial(q, k_loc.cuda(), v_loc.cuda(), sl_loc.cuda(), n, c.scale, m=m, l=l, o=o)
    return gathered


CASES = [
    # B, h_q, h_kv, d, seqlens, world, n_splits per rank, dtype
    (2, 64, 8, 128, [3000, 1234], 4, 4, "bf16"),
    (3, 32, 32, 128, [4096, 5, 0], 2, 8, "bf16"),
    (1, 16, 2, 64, [777], 8, 2, "bf16"),
    (2, 8, 2, 64, [300, 41], 3, 3, "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}_hq{c[1]}_w{c[5]}_n{c[6]}_{c[7]}" for c in CASES])
def test_sharded_merge_matches_oracle_and_single_gpu(gk, case):
    from gqa_split_kv_decode_b200 import sharded
    B, hq, hkv, d, seqlens, world, n, dtype = case
    w = random_case(B, hq, hkv, d, seqlens, dtype=dtype, seed=sum(seqlens) % 997)
    c = w.cfg
    gathered = _gathered(gk, w, world, n)
    out = sharded.merge_gathered(gathered, B, hq, n, d)
    torch.cuda.synchronize()
    assert gk.get_status() == 0
    ref = oracle.attn(w.q, w.k, w.v, w.seqlens, hq, hkv, c.scale).reshape(B, hq, d)
    got = out.double().cpu().numpy()
    atol, rtol = TOL[dtype]
    assert np.isfinite(got).all()
    assert (np.abs(got - ref) <= atol + rtol * np.abs(ref)).all()
    # the ranked merge is mlo_merge over the rank-major concatenation, bit for bit
    parts = [sharded.triplet_views(gathered[r], B, hq, n, d) for r in range(world)]
    M = torch.cat([p[0] for p in parts], dim=-1).contiguous()
    L = torch.cat([p[1] for p in parts], dim=-1).contiguous()
    O = torch.cat([p[2] for p in parts], dim=-2).contiguous()
    assert torch.equal(gk.mlo_merge(M, L, O), out)
    # and the separately gathered form of the binding agrees too
    Ms = torch.stack([p[0] for p in parts]).contiguous()
    Ls = torch.stack([p[1] for p in parts]).contiguous()
    Os = torch.stack([p[2] for p in parts]).contiguous()
    assert torch.equal(gk.mlo_merge_ranked(Ms, Ls, Os), out)


def test_sharded_decode_single_rank_is_partial_plus_merge(gk):
    from gqa_split_kv_decode_b200 import sharded
    w = random_case(2, 16, 2, 128, [900, 33], dtype="bf16", seed=3)
    c = w.cfg
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    out = sharded.sharded_decode(q, k, v, sl, 4, c.scale)
    m, l, o = gk.gqa_decode_partial(q, k, v, sl, 4, c.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, gk.mlo_merge(m, l, o))
    assert gk.get_status() == 0


def test_ranked_merge_rejects_overlapping_strides(gk):
    m = torch.zeros(2, 4, 3, device="cuda")
    o = torch.zeros(2, 4, 3, 64, device="cuda")
    out = torch.empty(4, 64, device="cuda")
    with pytest.raises(gk.GQADecodeError):
        gk.mlo_merge_ranked_raw(m, m, o, out, 4, 2, 3, 64, 11, 4 * 3 * 64)   # 11 < 4 * 3


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, case, q_out):
    """One rank of the sequence-sharded decode: its shard of every sequence,
    the library's partial triplets, the all-gather, the ranked merge."""
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import datetime

    import torch.distributed as dist

    import oracle as orc
    from gqa_split_kv_decode_b200 import sharded
    import gqa_split_kv_decode_b200 as gkr
    from workloads import random_case as rc

    B, hq, hkv, d, seqlens, n, dtype = case
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = rc(B, hq, hkv, d, seqlens, dtype=dtype, seed=sum(seqlens) % 991)
        c = w.cfg
        k_loc, v_loc, sl_loc = sharded.shard_packed_cache(w.k, w.v, w.seqlens, rank, world)
        out = sharded.sharded_decode(w.q.cuda(), k_loc.cuda(), v_loc.cuda(), sl_loc.cuda(), n, c.scale)
        torch.cuda.synchronize()
        status = gkr.get_status()
        ref = orc.attn(w.q, w.k, w.v, w.seqlens, hq, hkv, c.scale).reshape(B, hq, d)
        got = out.double().cpu().numpy()
        atol, rtol = TOL[dtype]
        excess = float((np.abs(got - ref) - (atol + rtol * np.abs(ref))).max())
        q_out.put((rank, status, excess, bool(np.isfinite(got).all())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", [
    (2, 64, 8, 128, [3000, 1234], 4, "bf16"),
    (3, 16, 2, 64, [0, 777, 5], 2, "f32"),
], ids=["llama70b_heads_bf16", "ragged_f32"])
def test_sharded_decode_two_ranks(gk, case):
    """The product function sharded_decode with two real ranks: two processes
    on cuda:0 joined by the gloo backend, whose all-gather moves the CUDA
    triplet buffers through the host.  No kernel of one rank waits on the
    other, so one GPU serves both.  Every rank must end with the full result
    (the oracle over the unsharded cache)."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, case, q_out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    res = sorted(q_out.get(timeout=10) for _ in range(2))
    assert [r[0] for r in res] == [0, 1]
    for _, status, excess, finite in res:
        assert status == 0 and finite
        assert excess <= 0.0, excess
