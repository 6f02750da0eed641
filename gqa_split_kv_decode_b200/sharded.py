"""Sequence-sharded decode across ranks: the method's own multi-GPU form.

kernbench "_attention_mesh_mlo.py" (module docstring and the kernel's
"One-shot local partial attention" / fan-out merge / "Final normalize"):
the single-token query is replicated on every rank, every sequence's KV
cache is cut along the sequence into one contiguous shard per rank, each
rank computes the (m, l, o) triplets of its shard, the triplets are
exchanged, and the log-sum-exp merge gives the exact full-sequence result.

The B200 form here: each rank's ``gqa_decode_partial`` writes its triplets
into one packed fp32 buffer, a single all-gather (NCCL over NVLink /
NVSwitch) brings every rank's buffer to every rank, and ``mlo_merge_ranked``
merges them straight out of the gathered buffer (no repacking).  Every rank
ends with the full output.  The exchange is B * h_q * n_splits * (d + 2)
floats per rank (266 KB for Llama-70B at 8 splits), so one collective per
step is the whole communication.

Host-side helpers (``shard_range``, ``shard_packed_cache``,
``triplet_layout``, ``exchange``) hold no attention arithmetic; the
computation is the library's kernels.
"""
from __future__ import annotations

import torch

from . import gqa_decode_partial, mlo_merge_ranked_raw, _default_scale

__all__ = ["shard_range", "shard_packed_cache", "triplet_layout", "triplet_views", "exchange",
           "merge_gathered", "sharded_decode"]


def shard_range(S: int, rank: int, world: int) -> tuple[int, int]:
    """Keys [lo, hi) of a length-S sequence held by ``rank``: contiguous,
    in rank order, lengths differing by at most one."""
    if world < 1 or not 0 <= rank < world or S < 0:
        raise ValueError("need 0 <= rank < world and S >= 0")
    return (S * rank) // world, (S * (rank + 1)) // world


def shard_packed_cache(k, v, seqlens, rank: int, world: int):
    """This rank's slice of every sequence of a packed cache
    ([sum S_b, h_kv, d]); returns (k_local, v_local, seqlens_local), packed
    the same way.  A setup step: a serving system fills each rank's shard
    directly."""
    lens = [int(x) for x in seqlens.tolist()]
    ks, vs, local, off = [], [], [], 0
    for S in lens:
        lo, hi = shard_range(S, rank, world)
        ks.append(k[off + lo:off + hi])
        vs.append(v[off + lo:off + hi])
        local.append(hi - lo)
        off += S
    k_loc = torch.cat(ks) if ks else k[:0]
    v_loc = torch.cat(vs) if vs else v[:0]
    return k_loc.contiguous(), v_loc.contiguous(), torch.tensor(local, dtype=torch.int32,
                                                                 device=seqlens.device)


def _round4(x: int) -> int:
    return (x + 3) // 4 * 4


def triplet_layout(rows: int, n_splits: int, d: int) -> tuple[int, int, int, int]:
    """Float offsets of o, m, l inside one rank's packed triplet buffer and its
    length: o [rows][n][d] first, then m and l [rows][n], each segment
    padded to 16 bytes."""
    o_off = 0
    m_off = _round4(rows * n_splits * d)
    l_off = m_off + _round4(rows * n_splits)
    return o_off, m_off, l_off, l_off + _round4(rows * n_splits)


def triplet_views(buf, B: int, h_q: int, n_splits: int, d: int):
    """(m, l, o) views of one rank's packed buffer, shaped like
    gqa_decode_partial's outputs."""
    o_off, m_off, l_off, _ = triplet_layout(B * h_q, n_splits, d)
    n = B * h_q * n_splits
    return (buf[m_off:m_off + n].view(B, h_q, n_splits), buf[l_off:l_off + n].view(B, h_q, n_splits),
            buf[o_off:o_off + n * d].view(B, h_q, n_splits, d))


def exchange(mine, world: int, group=None):
    """All-gather of every rank's packed buffer into [world, len] (rank order).
    One collective; the identity when world == 1."""
    if world == 1:
        return mine.view(1, -1)
    import torch.distributed as dist
    gathered = torch.empty((world, mine.numel()), dtype=mine.dtype, device=mine.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(gathered.view(-1), mine, group=group)
    else:
        dist.all_gather(list(gathered.unbind(0)), mine, group=group)
    return gathered


def merge_gathered(gathered, B: int, h_q: int, n_splits: int, d: int, out=None):
    """mlo_merge_ranked over a gathered [world, len] buffer -> fp32 [B, h_q, d]."""
    world, length = gathered.shape
    o_off, m_off, l_off, _ = triplet_layout(B * h_q, n_splits, d)
    if out is None:
        out = torch.empty((B, h_q, d), dtype=torch.float32, device=gathered.device)
    flat = gathered.view(-1)
    return mlo_merge_ranked_raw(flat[m_off:], flat[l_off:], flat[o_off:], out, B * h_q, world,
                                n_splits, d, length, length)


def sharded_decode(q, k_local, v_local, seqlens_local, n_splits: int, scale=None, group=None,
                   out=None):
    """Decode attention over a sequence-sharded cache: this rank's partial
    triplets (n_splits per rank over its shard), one all-gather, the merge.
    Every rank returns the full fp32 [B, h_q, d] result.  Ranks must call it
    together (it holds a collective)."""
    world = 1
    if group is not None or (torch.distributed.is_available() and torch.distributed.is_initialized()):
        world = torch.distributed.get_world_size(group)
    B, h_q, d = q.shape
    _, _, _, length = triplet_layout(B * h_q, n_splits, d)
    mine = torch.empty(length, dtype=torch.float32, device=q.device)
    m, l, o = triplet_views(mine, B, h_q, n_splits, d)
    gqa_decode_partial(q, k_local, v_local, seqlens_local, n_splits, _default_scale(d, scale),
                       m=m, l=l, o=o)
    gathered = exchange(mine, world, group)
    return merge_gathered(gathered, B, h_q, n_splits, d, out)
