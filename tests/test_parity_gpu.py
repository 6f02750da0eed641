"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Tolerances (elementwise, allclose convention):
    bf16 inputs: |gpu - oracle| <= 2e-3 + 1e-2 * |oracle|
    fp32 inputs: |gpu - oracle| <= 1e-5 + 1e-5 * |oracle|
Triplets are compared as m (absolute, scaled by max(1, |m|)), l (relative)
and the split's normalised output o / l (the tolerance above).  The method's
pages fix no triplet tolerance; the bounds below are readings from fp32
rounding: a logit is an fp32 sum of d = 128 exact bf16 (or fp32) products,
off by at most about d * 2^-24 of its magnitude, so m is within 1e-5 of
max(1, |m|); l sums up to a few thousand fp32 exponentials (each off by
twice the logit error plus the exp2 rounding) in short sequential runs and a
shuffle tree, so its relative error stays below 1e-4 for bf16 inputs (and
1e-5 for the fp32 path).  Measured worst cases on B200 over the workloads and
edge cases: 4.9e-7 (m) and 1.3e-6 (l).
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import workloads
from workloads import CONFIGS, random_case, scaled

pytestmark = pytest.mark.gpu

TOL = {"bf16": (2e-3, 1e-2), "f32": (1e-5, 1e-5)}
M_TOL = {"bf16": 1e-5, "f32": 1e-5}
L_RTOL = {"bf16": 1e-4, "f32": 1e-5}


@pytest.fixture(scope="module")
def gk():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gqa_split_kv_decode_b200 as gk
    return gk


def dev(w):
    return (w.q.cuda(), w.k.cuda(), w.v.cuda(), w.seqlens.cuda())


def assert_close(got, ref, dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    atol, rtol = TOL[dtype]
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {err.size} outside tolerance; worst at {i}: "
                             f"gpu={got[i]!r} oracle={ref[i]!r} err={err[i]:.3e} bound={bound[i]:.3e}")


def assert_triplets(m, l, o, om, ol, oo, dtype, what=""):
    m = m.reshape(om.shape).astype(np.float64)
    l = l.reshape(ol.shape).astype(np.float64)
    o = o.reshape(oo.shape).astype(np.float64)
    empty = om == -np.inf
    assert np.array_equal(m == -np.inf, empty), f"{what}: empty splits differ"
    assert np.all(l[empty] == 0) and np.all(o[empty] == 0), f"{what}: empty split not (-inf, 0, 0)"
    full = ~empty
    dm = np.abs(m[full] - om[full]) / np.maximum(1.0, np.abs(om[full]))
    assert dm.max(initial=0) <= M_TOL[dtype], f"{what}: m off by {dm.max():.3e}"
    dl = np.abs(l[full] - ol[full]) / ol[full]
    assert dl.max(initial=0) <= L_RTOL[dtype], f"{what}: l off by {dl.max():.3e}"
    assert_close(o[full] / l[full][:, None], oo[full] / ol[full][:, None], dtype, what + " o/l")


def oracle_out(w, items=None):
    c = w.cfg
    ref = oracle.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale, items=items)
    return ref


def run_fused(gk, w, n_splits=None, chunk_len=None, max_seqlen=None):
    c = w.cfg
    q, k, v, sl = dev(w)
    if chunk_len:
        out = gk.gqa_decode_attn_chunked(q, k, v, sl, chunk_len,
                                         w.max_seqlen if max_seqlen is None else max_seqlen, c.scale)
    else:
        out = gk.gqa_decode_attn(q, k, v, sl, n_splits, c.scale)
    torch.cuda.synchronize()
    assert gk.get_status() == 0
    return out.cpu().numpy()


# ---------------------------------------------------------------- the configs

@pytest.mark.parametrize("name", ["tiny", "llama7b", "llama70b"])
def test_config_full_parity(gk, name):
    """Every output of the first three workloads at full size, in the
    launch configuration the benchmark times (fused, split by count)."""
    w = workloads.generate(CONFIGS[name])
    c = w.cfg
    got = run_fused(gk, w, n_splits=c.n_splits)
    ref = oracle_out(w).reshape(c.B, c.h_q, c.d)
    assert_close(got, ref, c.dtype, name)


@pytest.mark.parametrize("name", ["tiny", "llama7b", "llama70b"])
def test_config_partials_and_merge(gk, name):
    """Triplets of every split against the oracle's, and mlo_merge of the
    oracle's own triplets against the oracle's merge."""
    w = workloads.generate(CONFIGS[name])
    c = w.cfg
    q, k, v, sl = dev(w)
    m, l, o = gk.gqa_decode_partial(q, k, v, sl, c.n_splits, c.scale)
    om, ol, oo = oracle.partials(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale, n_splits=c.n_splits)
    assert_triplets(m.cpu().numpy(), l.cpu().numpy(), o.cpu().numpy(), om, ol, oo, c.dtype, name)
    # the merge kernel alone, fed the oracle's triplets rounded to fp32
    mt = torch.from_numpy(om.astype(np.float32)).cuda()
    lt = torch.from_numpy(ol.astype(np.float32)).cuda()
    ot = torch.from_numpy(oo.astype(np.float32)).cuda()
    merged = gk.mlo_merge(mt, lt, ot).cpu().numpy()
    ref = oracle.merge(om.astype(np.float32), ol.astype(np.float32), oo.astype(np.float32))
    assert_close(merged, ref, "f32", name + " mlo_merge")


def test_longctx_reduced(gk):
    """The 1M-key workload's structure (64 splits, N(0,1)/2) at 64K keys."""
    w = workloads.generate(scaled("longctx", S=65536 + 37))
    c = w.cfg
    got = run_fused(gk, w, n_splits=64)
    assert_close(got, oracle_out(w).reshape(c.B, c.h_q, c.d), "bf16", "longctx/64K")


def test_ragged_reduced(gk):
    """The ragged workload's structure (chunk 1024, 1% of v rows x10) at
    B = 12, S_b in [128, 6000]."""
    w = workloads.generate(scaled("ragged", B=12, S=6000))
    c = w.cfg
    got = run_fused(gk, w, chunk_len=1024)
    assert_close(got, oracle_out(w).reshape(c.B, c.h_q, c.d), "bf16", "ragged/small")
    q, k, v, sl = dev(w)
    m, l, o = gk.gqa_decode_partial_chunked(q, k, v, sl, 1024, w.max_seqlen, c.scale)
    om, ol, oo = oracle.partials(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale, chunk_len=1024)
    assert_triplets(m.cpu().numpy(), l.cpu().numpy(), o.cpu().numpy(), om, ol, oo, "bf16", "ragged chunks")


@pytest.mark.parametrize("name", ["longctx", "ragged"])
def test_full_size_every_row(gk, name):
    """The two large workloads (about 4.3 and 4.8 GB of K/V) at full size, in
    the launch configuration the benchmark times; every output element of
    every (b, h) row against the oracle (a full fp64 pass takes a few seconds
    on the host's cores)."""
    w = workloads.generate(CONFIGS[name])
    c = w.cfg
    if c.chunk_len:
        got = run_fused(gk, w, chunk_len=c.chunk_len)
    else:
        got = run_fused(gk, w, n_splits=c.n_splits)
    ref = oracle_out(w).reshape(c.B, c.h_q, c.d)
    assert_close(got, ref, "bf16", name + " full size")


# ---------------------------------------------------------------- edge cases

EDGE = [
    # B, h_q, h_kv, d, seqlens, n_splits
    (6, 8, 2, 128, [0, 1, 7, 16, 33, 1000], 4),
    (6, 8, 2, 128, [0, 1, 7, 16, 33, 1000], 16),
    (3, 8, 2, 64, [17, 255, 3], 8),
    (2, 4, 4, 128, [300, 5], 3),          # MHA, G = 1
    (2, 8, 4, 128, [129, 64], 2),         # G = 2
    (2, 16, 4, 64, [90, 1], 5),           # G = 4
    (1, 16, 1, 128, [777], 7),            # G = 16: one 16-head block
    (1, 32, 1, 128, [500], 6),            # G = 32: two head blocks
    (2, 24, 2, 64, [100, 40], 3),         # G = 12: 16-head block, 4 padded
    (2, 12, 4, 128, [50, 70], 4),         # G = 3: padded 8-head block
    (1, 8, 1, 128, [5], 64),              # more splits than keys
    (1, 8, 1, 128, [5000], 1),            # one split
    (3, 8, 8, 64, [0, 0, 0], 4),          # every sequence empty
    (2, 8, 2, 128, [5000, 3], 1024),      # the most splits a call takes
    (300, 8, 2, 64, [(37 * i) % 61 for i in range(300)], 2),   # many short sequences
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("case", EDGE, ids=[f"B{c[0]}_hq{c[1]}_hkv{c[2]}_d{c[3]}_n{c[5]}_{i}" for i, c in enumerate(EDGE)])
def test_edge_cases(gk, case, dtype):
    B, hq, hkv, d, seqlens, n = case
    w = random_case(B, hq, hkv, d, seqlens, dtype=dtype, seed=zlib.crc32(repr((case, dtype)).encode()) % 10000)
    c = w.cfg
    got = run_fused(gk, w, n_splits=n)
    ref = oracle_out(w).reshape(B, hq, d)
    assert_close(got, ref, dtype, f"fused {case}")
    q, k, v, sl = dev(w)
    m, l, o = gk.gqa_decode_partial(q, k, v, sl, n, c.scale)
    om, ol, oo = oracle.partials(w.q, w.k, w.v, w.seqlens, hq, hkv, c.scale, n_splits=n)
    assert_triplets(m.cpu().numpy(), l.cpu().numpy(), o.cpu().numpy(), om, ol, oo, dtype, f"partial {case}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("chunk", [1, 16, 100, 1024])
def test_chunked_edges(gk, chunk, dtype):
    seqlens = [0, 1, 99, 100, 101, 1023, 1024]
    w = random_case(7, 8, 2, 128, seqlens, dtype=dtype, seed=chunk)
    c = w.cfg
    if -(-w.max_seqlen // chunk) > 1024:
        pytest.skip("more than 1024 chunks")
    got = run_fused(gk, w, chunk_len=chunk)
    assert_close(got, oracle_out(w).reshape(7, 8, 128), dtype, f"chunked {chunk}")


def test_dominant_logit_and_large_values(gk):
    """A logit far above the rest returns that key's V row; large V values
    stay within tolerance (closed form, no oracle)."""
    w = random_case(1, 8, 1, 128, [2000], dtype="bf16", seed=5)
    q = w.q.clone()
    k = w.k.clone()
    v = w.v.clone() * 30
    k[1234, 0, :] = (q[0, :, :].float().sum(0) * 4).to(torch.bfloat16)   # huge logit for all 8 heads
    w2 = workloads.Workload(w.cfg, q, k, v.to(torch.bfloat16), w.seqlens)
    got = run_fused(gk, w2, n_splits=8)
    ref = oracle_out(w2).reshape(1, 8, 128)
    assert_close(got, ref, "bf16", "dominant")
    row = v[1234, 0].double().numpy()
    assert np.allclose(got[0], np.broadcast_to(row, (8, 128)), atol=2e-3, rtol=1e-2)


# ------------------------------------------------------- exactness properties

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fused_matches_partial_then_merge(gk, dtype):
    """The fused call and partial + mlo_merge are two groupings of the same
    exact merge: they agree to fp32 rounding (bitwise on the fp32 path,
    which shares the per-split kernel)."""
    w = random_case(3, 64, 8, 128, [3000, 17, 900], dtype=dtype, seed=40)
    c = w.cfg
    q, k, v, sl = dev(w)
    fused = gk.gqa_decode_attn(q, k, v, sl, 8, c.scale)
    m, l, o = gk.gqa_decode_partial(q, k, v, sl, 8, c.scale)
    merged = gk.mlo_merge(m, l, o)
    if dtype == "f32":
        assert torch.equal(fused, merged)
    else:
        assert torch.allclose(fused, merged, atol=1e-5, rtol=1e-4)


def test_deterministic_and_workspace_reuse(gk):
    """Repeated calls on one workspace give bit-identical results (the split
    order of the merge is fixed and the tickets reset themselves)."""
    w = workloads.generate(scaled("llama70b", B=3, S=2500))
    c = w.cfg
    q, k, v, sl = dev(w)
    ws = torch.zeros(gk.workspace_size(c.B, c.h_q, c.h_kv, c.d, 8), dtype=torch.uint8, device="cuda")
    outs = [gk.gqa_decode_attn(q, k, v, sl, 8, c.scale, workspace=ws).clone() for _ in range(4)]
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    tickets = ws[: c.B * c.h_kv * 4].view(torch.int32)
    assert int(tickets.abs().sum()) == 0


def test_side_stream_and_library_workspace(gk):
    w = random_case(2, 8, 2, 128, [333, 1000], seed=3)
    c = w.cfg
    q, k, v, sl = dev(w)
    ref = oracle_out(w).reshape(2, 8, 128)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = gk.gqa_decode_attn(q, k, v, sl, 4, c.scale)
    s.synchronize()
    assert_close(out.cpu().numpy(), ref, "bf16", "side stream")


def test_binding_rejects_bad_tensors(gk):
    w = random_case(1, 8, 2, 128, [10], seed=4)
    q, k, v, sl = dev(w)
    with pytest.raises(ValueError):
        gk.gqa_decode_attn(q.float(), k, v, sl, 2)
    with pytest.raises(ValueError):
        gk.gqa_decode_attn(q, k, v, sl.long(), 2)
    with pytest.raises(ValueError):
        gk.gqa_decode_attn(q.transpose(0, 1), k, v, sl, 2)
    with pytest.raises(gk.GQADecodeError) as e:
        gk.gqa_decode_attn(q, k, v, sl, -1)
    assert e.value.status == 1


# ---------------------------------------------------------- device status

def test_negative_seqlen_reported(gk):
    w = random_case(2, 8, 2, 128, [10, 20], seed=6)
    q, k, v, sl = dev(w)
    sl[0] = -5
    out = gk.gqa_decode_attn(q, k, v, sl, 4, w.cfg.scale)
    assert gk.get_status() == gk.ERR_DEVICE_SEQLEN
    assert torch.all(out[0] == 0)
    assert gk.get_status() == 0  # cleared


def test_seqlen_over_max_reported(gk):
    w = random_case(1, 8, 2, 128, [3000], seed=7)
    q, k, v, sl = dev(w)
    gk.gqa_decode_attn_chunked(q, k, v, sl, 1024, 2048, w.cfg.scale)
    assert gk.get_status() == gk.ERR_DEVICE_SEQLEN
    assert gk.get_status() == 0


def test_bounded_wait_times_out_without_hanging(gk):
    """A wait that nothing ever satisfies ends after its bound and reports
    GQA_ERR_DEVICE_TIMEOUT; the context stays usable."""
    gk.selftest_wait_timeout(2_000_000)  # 2 ms
    assert gk.get_status() == gk.ERR_DEVICE_TIMEOUT
    assert gk.get_status() == 0
    w = random_case(1, 8, 2, 128, [100], seed=8)
    got = run_fused(gk, w, n_splits=2)
    assert_close(got, oracle_out(w).reshape(1, 8, 128), "bf16", "after timeout")
