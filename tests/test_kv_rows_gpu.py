"""The packed cache's row count (kv_rows) through the C ABI, against the
fp64 oracle.

Given kv_rows, no cache row at or past it is read: a batch whose lengths
run past the cache reads those rows as zero and reports
GQA_ERR_DEVICE_SEQLEN (the tensors here hold every row the lengths name, so
nothing outside them is touched either way).  kv_rows = -1 (not given)
turns the clip and the bf16 kernels' early L2 prefetch off; the result is
the same.  Each case names the launch plan it reaches.
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


def raw_fused(gk, w, kv_rows, n_splits):
    """gqa_decode_attn through the raw ctypes entry point with an explicit kv_rows."""
    c = w.cfg
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    B, h_q, d = q.shape
    h_kv = k.shape[1]
    out = torch.empty(B, h_q, d, device="cuda")
    ws = torch.zeros(gk.workspace_size(B, h_q, h_kv, d, n_splits), dtype=torch.uint8, device="cuda")
    dt = gk.BF16 if q.dtype == torch.bfloat16 else gk.F32
    rc = gk._attn(q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(), kv_rows, out.data_ptr(),
                  B, h_q, h_kv, d, n_splits, c.scale, dt, ws.data_ptr(), ws.numel(),
                  torch.cuda.current_stream().cuda_stream)
    assert rc == 0, rc
    torch.cuda.synchronize()
    return out.cpu().numpy()


def raw_partial(gk, w, kv_rows, n_splits):
    c = w.cfg
    q, k, v, sl = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda()
    B, h_q, d = q.shape
    h_kv = k.shape[1]
    m = torch.empty(B, h_q, n_splits, device="cuda")
    l = torch.empty_like(m)
    o = torch.empty(B, h_q, n_splits, d, device="cuda")
    dt = gk.BF16 if q.dtype == torch.bfloat16 else gk.F32
    rc = gk._partial(q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(), kv_rows, m.data_ptr(),
                     l.data_ptr(), o.data_ptr(), B, h_q, h_kv, d, n_splits, c.scale, dt,
                     torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    return m.cpu().numpy(), l.cpu().numpy(), o.cpu().numpy()


def assert_close(got, ref, dtype, what):
    atol, rtol = TOL[dtype]
    err = np.abs(np.asarray(got, np.float64) - ref)
    bound = atol + rtol * np.abs(ref)
    assert np.all(err <= bound), f"{what}: worst excess {np.max(err - bound):.3e}"


# (B, h_q, h_kv, d, seqlens, n_splits, the fused plan)
PLANS = [
    (2, 8, 2, 128, [100, 200], 4, "one_wave"),
    (1, 32, 32, 128, [1000], 8, "one_wave"),
    (8, 64, 8, 128, [200] * 8, 8, "persistent"),
    (64, 32, 8, 64, [(97 * i) % 180 + 20 for i in range(64)], 8, "many_waves"),
]


@pytest.mark.parametrize("case", PLANS, ids=[p[-1] + f"_B{p[0]}" for p in PLANS])
def test_kv_rows_not_given_matches_oracle(gk, case):
    """kv_rows = -1: no clip, no early prefetch; fused and partial results
    match the oracle as with kv_rows given."""
    B, hq, hkv, d, seqlens, n, plan = case
    assert gk.fused_plan(B, hq, hkv, d, n) == plan
    w = random_case(B, hq, hkv, d, seqlens, dtype="bf16", seed=len(seqlens) + n)
    ref = oracle.attn(w.q, w.k, w.v, w.seqlens, hq, hkv, w.cfg.scale).reshape(B, hq, d)
    for kv_rows in (-1, sum(seqlens)):
        assert_close(raw_fused(gk, w, kv_rows, n), ref, "bf16", f"fused kv_rows={kv_rows}")
        assert gk.get_status() == 0
    om, ol, oo = oracle.partials(w.q, w.k, w.v, w.seqlens, hq, hkv, w.cfg.scale, n_splits=n)
    m, l, o = raw_partial(gk, w, -1, n)
    m, l, o = m.reshape(om.shape), l.reshape(ol.shape), o.reshape(oo.shape)
    full = om > -np.inf
    assert np.array_equal(m > -np.inf, full)
    assert_close((o / np.where(full, l, 1)[..., None])[full], (oo / np.where(full, ol, 1)[..., None])[full],
                 "bf16", "partial o/l, kv_rows=-1")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("case", PLANS[::2], ids=[p[-1] for p in PLANS[::2]])
def test_rows_past_kv_rows_read_as_zero(gk, case, dtype):
    """Lengths that run past kv_rows: the rows from kv_rows on read as zero
    (the oracle on the cache with those rows zeroed) and the status word
    reports GQA_ERR_DEVICE_SEQLEN."""
    B, hq, hkv, d, seqlens, n, plan = case
    w = random_case(B, hq, hkv, d, seqlens, dtype=dtype, seed=11 + n)
    total = sum(seqlens)
    kv_rows = total - 37 - total // 5  # cuts into the last sequences, not on a tile edge
    kz, vz = w.k.clone(), w.v.clone()
    kz[kv_rows:] = 0
    vz[kv_rows:] = 0
    ref = oracle.attn(w.q, kz, vz, w.seqlens, hq, hkv, w.cfg.scale).reshape(B, hq, d)
    got = raw_fused(gk, w, kv_rows, n)
    assert gk.get_status() == gk.ERR_DEVICE_SEQLEN
    assert gk.get_status() == 0
    assert_close(got, ref, dtype, f"clipped at {kv_rows} of {total} rows")
