"""Append-and-attend (gqa_decode_attn_append) against the oracle.

The cache is padded [B, cap, h_kv, d]; every row past a sequence's length is
filled with NaN, so a kernel that lets any of them into the result fails.
The oracle attends over the cached rows plus the new token, packed.
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


def _padded_case(B, hq, hkv, d, seqlens, cap, dtype, seed):
    """Packed random rows for each sequence's cache plus one new token, laid
    out in a NaN-filled padded cache."""
    full = [min(s + 1, cap) for s in seqlens]              # cached rows + the new one (if room)
    w = random_case(B, hq, hkv, d, full, dtype=dtype, seed=seed)
    dt = w.k.dtype
    kc = torch.full((B, cap, hkv, d), float("nan"), dtype=dt)
    vc = torch.full((B, cap, hkv, d), float("nan"), dtype=dt)
    kn = torch.empty((B, hkv, d), dtype=dt)
    vn = torch.empty((B, hkv, d), dtype=dt)
    off = 0
    for b, s in enumerate(seqlens):
        n = full[b]
        rows_k, rows_v = w.k[off:off + n], w.v[off:off + n]
        if s < cap:  # last packed row is the new token
            kc[b, :s] = rows_k[:s]
            vc[b, :s] = rows_v[:s]
            kn[b], vn[b] = rows_k[s], rows_v[s]
        else:        # no room: all rows cached, the new token is never attended
            kc[b, :n] = rows_k
            vc[b, :n] = rows_v
            kn[b] = torch.randn(hkv, d).to(dt)
            vn[b] = torch.randn(hkv, d).to(dt)
        off += n
    return w, kc, vc, kn, vn


def _check(got, w, dtype):
    c = w.cfg
    ref = oracle.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale).reshape(c.B, c.h_q, c.d)
    got = got.double().cpu().numpy()
    assert np.isfinite(got).all()
    atol, rtol = TOL[dtype]
    err = np.abs(got - ref)
    assert (err <= atol + rtol * np.abs(ref)).all(), float((err - atol - rtol * np.abs(ref)).max())


CASES = [
    # B, h_q, h_kv, d, seqlens, cap, n_splits, dtype
    (3, 16, 2, 128, [0, 5, 299], 300, 4, "bf16"),                  # one wave; last row fills the cap
    (4, 64, 8, 128, [1000, 15, 0, 600], 1100, 16, "bf16"),          # persistent plan
    (6, 64, 8, 64, [3, 0, 480, 33, 16, 1], 500, 64, "bf16"),        # many waves, d = 64
    (2, 32, 2, 128, [700, 9], 800, 5, "bf16"),                      # 16-head blocks
    (2, 8, 2, 64, [7, 50], 100, 3, "f32"),                          # fp32 path
    (3, 4, 4, 128, [0, 17, 64], 65, 2, "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}_hq{c[1]}_hkv{c[2]}_d{c[3]}_n{c[6]}_{c[7]}" for c in CASES])
def test_append_then_attend(gk, case):
    B, hq, hkv, d, seqlens, cap, n, dtype = case
    w, kc, vc, kn, vn = _padded_case(B, hq, hkv, d, seqlens, cap, dtype, seed=sum(seqlens) % 1000)
    q = w.q.cuda()
    kc_d, vc_d, kn_d, vn_d = kc.cuda(), vc.cuda(), kn.cuda(), vn.cuda()
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    out = gk.gqa_decode_attn_append(q, kn_d, vn_d, kc_d, vc_d, sl, n, w.cfg.scale)
    torch.cuda.synchronize()
    assert gk.get_status() == 0
    _check(out, w, dtype)
    # the new rows landed at row S_b; every other row is as it was
    kc_after, vc_after = kc_d.cpu(), vc_d.cpu()
    for b, s in enumerate(seqlens):
        assert torch.equal(kc_after[b, s], kn[b]) and torch.equal(vc_after[b, s], vn[b])
        kc[b, s], vc[b, s] = kn[b], vn[b]
    assert torch.equal(kc_after.view(torch.int16 if kc.dtype == torch.bfloat16 else torch.int32),
                       kc.view(torch.int16 if kc.dtype == torch.bfloat16 else torch.int32))
    assert torch.equal(vc_after.view(torch.int16 if vc.dtype == torch.bfloat16 else torch.int32),
                       vc.view(torch.int16 if vc.dtype == torch.bfloat16 else torch.int32))
    assert torch.equal(sl.cpu(), torch.tensor(seqlens, dtype=torch.int32))  # not advanced


def test_append_without_room_is_reported(gk):
    """S_b == cap: nothing is appended, the cached rows are attended and the
    status word says so."""
    seqlens, cap = [40, 64], 64
    w, kc, vc, kn, vn = _padded_case(2, 16, 2, 128, seqlens, cap, "bf16", seed=9)
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    kc_d, vc_d = kc.cuda(), vc.cuda()
    out = gk.gqa_decode_attn_append(w.q.cuda(), kn.cuda(), vn.cuda(), kc_d, vc_d, sl, 4, w.cfg.scale)
    assert gk.get_status() == gk.ERR_DEVICE_SEQLEN
    assert gk.get_status() == 0
    _check(out, w, "bf16")
    assert torch.isnan(kc_d[0, 41:].float()).all()           # nothing written past the new row
    assert torch.equal(kc_d[1].cpu(), kc[1])                  # the full sequence is untouched


def test_append_steps_match_a_growing_cache(gk):
    """Three decode steps: append, advance seqlens, repeat -- each step's output
    equals plain attention over the grown cache."""
    B, hq, hkv, d, cap = 2, 16, 2, 128, 64
    torch.manual_seed(0)
    kc = torch.randn(B, cap, hkv, d).to(torch.bfloat16).cuda()
    vc = torch.randn(B, cap, hkv, d).to(torch.bfloat16).cuda()
    sl = torch.tensor([10, 30], dtype=torch.int32, device="cuda")
    for step in range(3):
        q = torch.randn(B, hq, d).to(torch.bfloat16).cuda()
        kn = torch.randn(B, hkv, d).to(torch.bfloat16).cuda()
        vn = torch.randn(B, hkv, d).to(torch.bfloat16).cuda()
        out = gk.gqa_decode_attn_append(q, kn, vn, kc, vc, sl, 2)
        sl += 1
        lens = sl.cpu().tolist()
        kp = torch.cat([kc[b, :lens[b]] for b in range(B)]).cpu()
        vp = torch.cat([vc[b, :lens[b]] for b in range(B)]).cpu()
        ref = oracle.attn(q.cpu(), kp, vp, lens, hq, hkv, 1 / np.sqrt(d)).reshape(B, hq, d)
        err = np.abs(out.double().cpu().numpy() - ref)
        assert (err <= 2e-3 + 1e-2 * np.abs(ref)).all()
    assert gk.get_status() == 0
