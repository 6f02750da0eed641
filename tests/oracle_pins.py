"""Pins for the CPU oracle: facts fixed by the pages and by mathematics.

Each ``pin_*`` takes an oracle handle (``oracle.Oracle``) and raises
AssertionError when the oracle disagrees with something that does not come
from the oracle itself: a hand-worked example, a 50-digit brute force, a
closed form, a library routine, or an invariant of the method.  The same pins
run against copies of the oracle with a planted mistake, each of which must
fail at least one of them.
"""
from __future__ import annotations

import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import torch

from workloads import random_case

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "merge_example.txt")


# --------------------------------------------------------------------------
# helpers (no attention arithmetic of the oracle's kind lives here)

def _golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            name, *rest = line.split()
            out = []
            for tok in rest:
                if tok.startswith("ln:"):
                    out.append(("ln", Fraction(tok[3:])))
                else:
                    out.append(Fraction(tok))
            vals[name] = out
    return vals


def _num(x):
    if isinstance(x, tuple):
        return math.log(float(x[1]))
    return float(x)


def _exact(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 values of a fp32 / bf16 tensor."""
    return t.to(torch.float64).numpy()


def _offsets(seqlens):
    off = [0]
    for s in seqlens:
        off.append(off[-1] + int(s))
    return off


# --------------------------------------------------------------------------
# pins

def pin_worked_example(orc):
    """Hand-worked merge example (tests/golden/merge_example.txt)."""
    g = _golden()
    logits = [_num(x) for x in g["logits"]]
    q = torch.tensor([[[1.0, 0.0]]], dtype=torch.float32)
    k = torch.tensor([[[s, 0.0]] for s in logits], dtype=torch.float32)
    v = torch.tensor([[[float(a) for a in g[f"v{j}"]]] for j in range(4)], dtype=torch.float32)
    sl = [4]
    m, l, o = orc.partials(q, k, v, sl, 1, 1, 1.0, n_splits=2)
    assert np.allclose(m[0], [_num(g["m_A"][0]), _num(g["m_B"][0])], rtol=0, atol=1e-6), m
    assert np.allclose(l[0], [float(g["l_A"][0]), float(g["l_B"][0])], rtol=1e-6, atol=0), l
    assert np.allclose(o[0, 0], [float(x) for x in g["o_A"]], rtol=1e-6, atol=1e-7), o
    assert np.allclose(o[0, 1], [float(x) for x in g["o_B"]], rtol=1e-6, atol=1e-7), o
    O_ref = [float(x) for x in g["O"]]
    # merge of the exact triplets
    mm = np.array([[_num(g["m_A"][0]), _num(g["m_B"][0])]])
    ll = np.array([[float(g["l_A"][0]), float(g["l_B"][0])]])
    oo = np.array([[[float(x) for x in g["o_A"]], [float(x) for x in g["o_B"]]]])
    out = orc.merge(mm, ll, oo)
    assert np.allclose(out[0], O_ref, rtol=1e-14, atol=0), out
    # the order of the splits does not matter, nor does an empty split
    out_r = orc.merge(mm[:, ::-1].copy(), ll[:, ::-1].copy(), oo[:, ::-1].copy())
    assert np.allclose(out_r[0], O_ref, rtol=1e-14, atol=0), out_r
    mm3 = np.array([[mm[0, 0], -np.inf, mm[0, 1]]])
    ll3 = np.array([[ll[0, 0], 0.0, ll[0, 1]]])
    oo3 = np.concatenate([oo[:, :1], np.zeros((1, 1, 2)), oo[:, 1:]], axis=1)
    out3 = orc.merge(mm3, ll3, oo3)
    assert np.allclose(out3[0], O_ref, rtol=1e-14, atol=0), out3
    # direct attention through the oracle's unsplit path
    full = orc.attn(q, k, v, sl, 1, 1, 1.0)
    assert np.allclose(full[0], O_ref, rtol=1e-6, atol=1e-7), full
    # the merged triplet itself: one split holding all four keys
    m1, l1, o1 = orc.partials(q, k, v, sl, 1, 1, 1.0, n_splits=1)
    assert abs(m1[0, 0] - _num(g["m_merged"][0])) <= 1e-6
    assert abs(l1[0, 0] - float(g["l_merged"][0])) <= 1e-6
    assert np.allclose(o1[0, 0], [float(x) for x in g["o_merged"]], rtol=1e-6, atol=1e-7)


def _decimal_case(w, items_splits=2):
    """50-digit brute force: exp without max subtraction, then the triplet
    of each contiguous split formed from exact sums."""
    getcontext().prec = 50
    c = w.cfg
    q = _exact(w.q)
    k = _exact(w.k)
    v = _exact(w.v)
    off = _offsets(w.seqlens.tolist())
    G = c.h_q // c.h_kv
    out = {}
    parts = {}
    for b in range(c.B):
        S = int(w.seqlens[b])
        for h in range(c.h_q):
            kvh = h // G
            s = []
            for j in range(S):
                acc = Decimal(0)
                for t in range(c.d):
                    acc += Decimal(float(q[b, h, t])) * Decimal(float(k[off[b] + j, kvh, t]))
                s.append(acc * Decimal(c.scale))
            e = [x.exp() for x in s]
            den = sum(e, Decimal(0))
            num = [sum((e[j] * Decimal(float(v[off[b] + j, kvh, t])) for j in range(S)), Decimal(0))
                   for t in range(c.d)]
            out[(b, h)] = [float(x / den) if S else 0.0 for x in num]
            L = -(-S // items_splits) if S else 0
            trip = []
            for i in range(items_splits):
                lo, hi = min(i * L, S), min((i + 1) * L, S)
                if hi <= lo:
                    trip.append((-math.inf, 0.0, [0.0] * c.d))
                    continue
                mx = max(s[lo:hi])
                sc = (-mx).exp()
                lsum = sum(e[lo:hi], Decimal(0)) * sc
                osum = [sum((e[j] * Decimal(float(v[off[b] + j, kvh, t])) for j in range(lo, hi)),
                            Decimal(0)) * sc for t in range(c.d)]
                trip.append((float(mx), float(lsum), [float(x) for x in osum]))
            parts[(b, h)] = trip
    return out, parts


def pin_decimal_bruteforce(orc):
    """Tiny inputs against a 50-digit Decimal brute force."""
    cases = [
        dict(B=2, h_q=2, h_kv=1, d=2, seqlens=[3, 5], dtype="f32", seed=11),
        dict(B=2, h_q=4, h_kv=2, d=4, seqlens=[1, 2], dtype="bf16", seed=12),
        dict(B=1, h_q=4, h_kv=1, d=4, seqlens=[5], dtype="bf16", seed=13, std=2.0),
        dict(B=3, h_q=2, h_kv=2, d=2, seqlens=[2, 0, 3], dtype="f32", seed=14),
    ]
    for cs in cases:
        w = random_case(**cs)
        c = w.cfg
        exact, parts = _decimal_case(w, items_splits=2)
        got = orc.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale)
        m, l, o = orc.partials(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale, n_splits=2)
        for idx, (b, h) in enumerate([(b, h) for b in range(c.B) for h in range(c.h_q)]):
            ref = np.array(exact[(b, h)])
            assert np.allclose(got[idx], ref, rtol=1e-12, atol=1e-13), (cs, b, h, got[idx], ref)
            for i, (mi, li, oi) in enumerate(parts[(b, h)]):
                if mi == -math.inf:
                    assert m[idx, i] == -np.inf and l[idx, i] == 0 and not np.any(o[idx, i]), (cs, b, h, i)
                else:
                    assert abs(m[idx, i] - mi) <= 1e-12 * max(1.0, abs(mi)), (cs, b, h, i)
                    assert abs(l[idx, i] - li) <= 1e-12 * li, (cs, b, h, i)
                    assert np.allclose(o[idx, i], oi, rtol=1e-12, atol=1e-13), (cs, b, h, i)


def pin_scale_zero_is_mean(orc):
    """scale = 0 makes every weight equal: O is the plain mean of V rows."""
    w = random_case(B=2, h_q=8, h_kv=2, d=64, seqlens=[37, 300], dtype="bf16", seed=21)
    c = w.cfg
    got = orc.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, 0.0)
    v = _exact(w.v)
    off = _offsets(w.seqlens.tolist())
    G = c.h_q // c.h_kv
    for b in range(c.B):
        for h in range(c.h_q):
            ref = v[off[b]:off[b + 1], h // G, :].mean(axis=0)
            assert np.allclose(got[b * c.h_q + h], ref, rtol=1e-12, atol=1e-14), (b, h)


def pin_constant_keys_is_mean(orc):
    """All keys of a kv head identical: O is the mean of that head's V rows."""
    w = random_case(B=1, h_q=4, h_kv=2, d=64, seqlens=[129], dtype="bf16", seed=22)
    w.k[:] = w.k[0:1]
    c = w.cfg
    got = orc.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale)
    v = _exact(w.v)
    for h in range(c.h_q):
        ref = v[:, h // 2, :].mean(axis=0)
        assert np.allclose(got[h], ref, rtol=1e-12, atol=1e-14), h


def pin_single_key(orc):
    """S_b = 1: the softmax weight is 1, so O is that key's V row."""
    w = random_case(B=3, h_q=4, h_kv=4, d=128, seqlens=[1, 1, 1], dtype="bf16", seed=23)
    c = w.cfg
    got = orc.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale)
    v = _exact(w.v)
    for b in range(3):
        for h in range(4):
            assert np.array_equal(got[b * 4 + h], v[b, h, :]), (b, h)


def pin_dominant_logit(orc):
    """One logit 200 above the rest: O is that key's V row (to e^-190)."""
    w = random_case(B=1, h_q=1, h_kv=1, d=8, seqlens=[50], dtype="f32", seed=24, std=0.1)
    w.q[:] = 0
    w.q[0, 0, 0] = 1.0
    w.k[17, 0, 0] = 200.0
    got = orc.attn(w.q, w.k, w.v, w.seqlens, 1, 1, 1.0)
    assert np.allclose(got[0], _exact(w.v)[17, 0], rtol=1e-14, atol=0), got


def pin_gqa_contiguous_mapping(orc):
    """V of kv head g held at the constant g + 1: O of query head h is
    floor(h / G) + 1 exactly (contiguous groups)."""
    w = random_case(B=2, h_q=8, h_kv=2, d=64, seqlens=[40, 9], dtype="bf16", seed=25)
    for g in range(2):
        w.v[:, g, :] = g + 1
    got = orc.attn(w.q, w.k, w.v, w.seqlens, 8, 2, w.cfg.scale)
    for b in range(2):
        for h in range(8):
            assert np.all(np.abs(got[b * 8 + h] - (h // 4 + 1)) < 1e-13), (b, h, got[b * 8 + h][:4])


def _sdpa_ref(w, scale):
    """torch's scaled_dot_product_attention in fp64 on the CPU, sequence by
    sequence, with each kv head repeated for its G consecutive query heads."""
    c = w.cfg
    G = c.h_q // c.h_kv
    off = _offsets(w.seqlens.tolist())
    outs = []
    for b in range(c.B):
        qb = w.q[b].double()[:, None, :]                              # [h_q, 1, d]
        kb = w.k[off[b]:off[b + 1]].double().permute(1, 0, 2)         # [h_kv, S, d]
        vb = w.v[off[b]:off[b + 1]].double().permute(1, 0, 2)
        kb = kb.repeat_interleave(G, dim=0)
        vb = vb.repeat_interleave(G, dim=0)
        ob = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, scale=scale)
        outs.append(ob[:, 0, :])
    return torch.cat(outs).numpy()


def pin_matches_library_sdpa(orc):
    """MHA and GQA against torch's fp64 scaled_dot_product_attention."""
    for cs in [dict(B=2, h_q=4, h_kv=4, d=64, seqlens=[100, 33], seed=26),
               dict(B=2, h_q=8, h_kv=2, d=128, seqlens=[257, 64], seed=27),
               dict(B=1, h_q=16, h_kv=1, d=64, seqlens=[80], seed=28)]:
        w = random_case(dtype="bf16", **cs)
        c = w.cfg
        got = orc.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale)
        ref = _sdpa_ref(w, c.scale)
        assert np.allclose(got, ref, rtol=1e-11, atol=1e-13), (cs, np.abs(got - ref).max())


def pin_partial_is_range_softmax(orc):
    """A split's triplet: m is the max logit of its keys, m + log(l) is their
    log-sum-exp, and o / l is the softmax-weighted mean of their V rows (all
    three from torch fp64 routines on that key range alone)."""
    w = random_case(B=2, h_q=4, h_kv=2, d=64, seqlens=[70, 5], dtype="bf16", seed=29)
    c = w.cfg
    n = 4
    m, l, o = orc.partials(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale, n_splits=n)
    off = _offsets(w.seqlens.tolist())
    for b in range(c.B):
        S = int(w.seqlens[b])
        L = -(-S // n)
        for h in range(c.h_q):
            g = h // 2
            for i in range(n):
                lo, hi = min(i * L, S), min((i + 1) * L, S)
                r = b * c.h_q + h
                if hi <= lo:
                    assert m[r, i] == -np.inf and l[r, i] == 0 and not o[r, i].any()
                    continue
                K = w.k[off[b] + lo:off[b] + hi, g].double()
                V = w.v[off[b] + lo:off[b] + hi, g].double()
                s = c.scale * (K @ w.q[b, h].double())
                assert abs(m[r, i] - s.max().item()) <= 1e-12
                assert abs(m[r, i] + math.log(l[r, i]) - torch.logsumexp(s, 0).item()) <= 1e-12
                ref = torch.softmax(s, 0) @ V
                assert np.allclose(o[r, i] / l[r, i], ref.numpy(), rtol=1e-11, atol=1e-13)


def pin_split_merge_invariance(orc):
    """Merging the triplets of any split count, chunking or split order gives
    the unsplit result."""
    w = random_case(B=3, h_q=8, h_kv=2, d=64, seqlens=[300, 7, 64], dtype="bf16", seed=30)
    c = w.cfg
    full = orc.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale)
    rng = np.random.default_rng(0)
    for kw in [dict(n_splits=1), dict(n_splits=2), dict(n_splits=3), dict(n_splits=7),
               dict(n_splits=64), dict(chunk_len=1), dict(chunk_len=5), dict(chunk_len=1024)]:
        m, l, o = orc.partials(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale, **kw)
        got = orc.merge(m, l, o)
        assert np.allclose(got, full, rtol=1e-12, atol=1e-14), kw
        perm = rng.permutation(m.shape[1])
        got_p = orc.merge(m[:, perm], l[:, perm], o[:, perm])
        assert np.allclose(got_p, full, rtol=1e-12, atol=1e-14), kw


def pin_empty_sequences(orc):
    """S_b = 0: every split is (-inf, 0, 0) and the output row is 0."""
    w = random_case(B=3, h_q=4, h_kv=1, d=64, seqlens=[0, 12, 0], dtype="bf16", seed=31)
    c = w.cfg
    full = orc.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale)
    assert not full[0:4].any() and not full[8:12].any()
    assert np.abs(full[4:8]).max() > 0
    m, l, o = orc.partials(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale, n_splits=3)
    assert np.all(m[0:4] == -np.inf) and not l[0:4].any() and not o[0:4].any()
    got = orc.merge(m, l, o)
    assert np.allclose(got, full, rtol=1e-12, atol=1e-14)


def pin_head_permutation(orc):
    """Permuting the query heads inside a group permutes the outputs."""
    w = random_case(B=1, h_q=8, h_kv=2, d=64, seqlens=[90], dtype="bf16", seed=32)
    c = w.cfg
    full = orc.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale)
    perm = [2, 0, 3, 1, 7, 5, 4, 6]
    q2 = w.q[:, perm, :].contiguous()
    got = orc.attn(q2, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale)
    assert np.array_equal(got, full[perm])


def _sdpa_causal_ref(q, k, v, seqlens, h_q, h_kv, scale):
    """torch's fp64 causal scaled_dot_product_attention, sequence by sequence,
    each kv head repeated for its consecutive query heads; rows in q's order."""
    G = h_q // h_kv
    off = _offsets(list(seqlens))
    outs = []
    for b in range(len(seqlens)):
        qb = q[off[b]:off[b + 1]].double().permute(1, 0, 2)                      # [h_q, S, d]
        kb = k[off[b]:off[b + 1]].double().permute(1, 0, 2).repeat_interleave(G, dim=0)
        vb = v[off[b]:off[b + 1]].double().permute(1, 0, 2).repeat_interleave(G, dim=0)
        ob = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, is_causal=True, scale=scale)
        outs.append(ob.permute(1, 0, 2).reshape(-1, q.shape[-1]))                 # [(S, h_q), d]
    return torch.cat(outs).numpy()


def _prefill_case(seqlens, h_q, h_kv, d, dtype, seed, std=1.0):
    """Packed q [sum S, h_q, d] plus k, v [sum S, h_kv, d]."""
    w = random_case(len(seqlens), h_q, h_kv, d, seqlens, dtype=dtype, seed=seed, std=std)
    rows = int(sum(seqlens))
    g = torch.Generator().manual_seed(seed + 7)
    q = (torch.randn(rows, h_q, d, generator=g) * std).to(w.k.dtype)
    return q, w.k, w.v, w.seqlens, w.cfg.scale


def pin_prefill_matches_library_causal_sdpa(orc):
    """Causal prefill against torch's fp64 causal SDPA (MHA and GQA)."""
    for seqlens, hq, hkv, d in [([33, 7], 4, 4, 64), ([40, 1, 17], 8, 2, 128)]:
        q, k, v, sl, scale = _prefill_case(seqlens, hq, hkv, d, "bf16", seed=sum(seqlens))
        got = orc.prefill(q, k, v, sl, hq, hkv, scale)
        ref = _sdpa_causal_ref(q, k, v, seqlens, hq, hkv, scale)
        assert np.allclose(got, ref, rtol=1e-11, atol=1e-13), np.abs(got - ref).max()


def pin_prefill_decimal_bruteforce(orc):
    """Tiny causal cases against a 50-digit Decimal brute force."""
    getcontext().prec = 50
    seqlens, hq, hkv, d = [3, 2], 4, 2, 4
    q, k, v, sl, scale = _prefill_case(seqlens, hq, hkv, d, "f32", seed=44)
    qx, kx, vx = _exact(q), _exact(k), _exact(v)
    off = _offsets(seqlens)
    items, ref = [], []
    for b, S in enumerate(seqlens):
        for i in range(S):
            for h in range(hq):
                g = h // (hq // hkv)
                s = []
                for j in range(i + 1):
                    acc = Decimal(0)
                    for t in range(d):
                        acc += Decimal(float(qx[off[b] + i, h, t])) * Decimal(float(kx[off[b] + j, g, t]))
                    s.append((acc * Decimal(scale)).exp())
                den = sum(s, Decimal(0))
                ref.append([float(sum((s[j] * Decimal(float(vx[off[b] + j, g, t])) for j in range(i + 1)),
                                      Decimal(0)) / den) for t in range(d)])
                items.append((b, h, i))
    got = orc.prefill(q, k, v, sl, hq, hkv, scale, items=items)
    assert np.allclose(got, np.array(ref), rtol=1e-12, atol=1e-13)


def pin_prefill_first_row_and_last_row(orc):
    """Position 0 attends only itself: O = v_0.  The last position of a
    sequence attends every key: it equals decode attention with that query."""
    seqlens, hq, hkv, d = [25, 9], 8, 2, 64
    q, k, v, sl, scale = _prefill_case(seqlens, hq, hkv, d, "bf16", seed=45)
    off = _offsets(seqlens)
    vx = _exact(v)
    got0 = orc.prefill(q, k, v, sl, hq, hkv, scale, items=[(b, h, 0) for b in range(2) for h in range(hq)])
    for b in range(2):
        for h in range(hq):
            assert np.array_equal(got0[b * hq + h], vx[off[b], h // 4])
    last = orc.prefill(q, k, v, sl, hq, hkv, scale,
                       items=[(b, h, seqlens[b] - 1) for b in range(2) for h in range(hq)])
    qd = torch.stack([q[off[b + 1] - 1] for b in range(2)])                     # [B, h_q, d]
    dec = orc.attn(qd, k, v, sl, hq, hkv, scale)
    assert np.allclose(last, dec, rtol=1e-13, atol=1e-15)


PINS = [pin_worked_example, pin_decimal_bruteforce, pin_scale_zero_is_mean,
        pin_constant_keys_is_mean, pin_single_key, pin_dominant_logit,
        pin_gqa_contiguous_mapping, pin_matches_library_sdpa, pin_partial_is_range_softmax,
        pin_split_merge_invariance, pin_empty_sequences, pin_head_permutation,
        pin_prefill_matches_library_causal_sdpa, pin_prefill_decimal_bruteforce,
        pin_prefill_first_row_and_last_row]
