"""Benchmark: fused split-KV GQA decode attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

--config llama70b_prefill2k | prefill_ragged measures the causal prefill
kernel instead (one step = one gqa_prefill_attn call; metric TFLOP/s of the
attended (query, key) pairs against the measured bf16 tensor-core peak).

One step = one call of the fused decode (every step of the path: split
assignment, TMA-fed K/V stream, logits, online softmax, PV, triplets and the
log-sum-exp merge) over one batch of the workload, inputs resident in HBM.
Metric (the headline of the method's target): KV bytes read per second
(GB/s), with us/call and the fraction of measured HBM bandwidth.  Between
timed steps the inputs rotate among copies totalling >= 1 GiB so no step
reads K/V from L2.  Multi-GPU runs are independent replicas (one per rank,
weak scaling); time is the max over ranks of CUDA-event time.

--sharded (decode workloads) runs the method's multi-rank form: each rank
holds a contiguous 1/N slice of every sequence's cache, computes its partial
triplets, one all-gather exchanges them and every rank merges (strong
scaling: the value is the whole cache's KV bytes per second).

--impl reference times the CPU oracle (fp64, every host core) on a bounded
sample of the same workload per step; the GPU is not used.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "GQA decode attention: KV-read HBM GB/s and % of B200 peak; µs/call"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2**20
ROTATE_TOTAL = 1 << 30
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "decode_tc_bf16_persist_llama70b.md")
PREFILL_PROFILE = os.path.join(ROOT, "profiles", "prefill_tc_bf16_llama70b_prefill2k.md")
PREFILL_METRIC = "GQA causal prefill attention: TFLOP/s of attended (query, key) pairs and % of B200 bf16 peak; µs/call"
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--config", default="llama70b",
                   choices=sorted(workloads.CONFIGS) + sorted(workloads.PREFILL_CONFIGS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-clocks", action="store_true")
    p.add_argument("--seq-len", type=int, default=None,
                   help="decode: override the workload's S (the ragged workload's upper bound), "
                        "e.g. a smaller case of the same structure for an ncu capture")
    p.add_argument("--batch", type=int, default=None, help="decode: override the workload's B")
    p.add_argument("--no-graph", action="store_true",
                   help="time the K steps as direct calls only (no CUDA-graph replay)")
    p.add_argument("--no-hold", action="store_true",
                   help="start the timed region on an idle GPU (no device-side hold before the "
                        "start event), so the host's first submission falls inside it")
    p.add_argument("--no-per-config", action="store_true",
                   help="decode: time only the headline workload (skip the per_config object)")
    p.add_argument("--seed", type=int, default=None,
                   help="seed of the synthetic inputs (default: the workload's own, 1000 + config "
                        "index for decode, 2000 + index for prefill)")
    p.add_argument("--sharded", action="store_true",
                   help="decode with every sequence's KV cache split over the ranks (partial triplets, "
                        "one all-gather, merge) instead of independent replicas")
    return p.parse_args(argv)


# ----------------------------------------------------------------- helpers

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# The sources each profiled kernel is compiled from (a committed ncu summary
# stays valid while none of them changes).
DECODE_SOURCES = ("device_common.cuh", "decode_tc.cuh", "decode_persist.cuh", "split_merge.cuh")
PREFILL_SOURCES = ("device_common.cuh", "tcgen05.cuh", "prefill_tc.cuh")


def kernel_source_hash(names=DECODE_SOURCES) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gqa_split_kv_decode_b200", "csrc")
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def measured_bf16_peak():
    """(burst, sustained, source) bf16 dense TFLOP/s."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


def profiled_traffic(config: str, summary: str = PROFILE_SUMMARY, sources=DECODE_SOURCES):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources and this workload (else None)."""
    try:
        text = open(summary).read()
    except OSError:
        return None
    src = re.search(r"kernel_source_hash:\s*(\w+)", text)
    wl = re.search(r"workload:\s*(\w+)", text)
    tr = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not (src and wl and tr) or src.group(1) != kernel_source_hash(sources) or wl.group(1) != config:
        return None
    return int(tr.group(1))


class ClockSampler:
    """nvidia-smi samples (every 200 ms) of SM clock and throttle reasons."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, window=None):
        """Median SM clock and the throttle reasons seen in the samples taken
        during `window` (host wall times (t0, t1)), widened by one sampling
        period on each side so a region shorter than the period still has
        its neighbouring samples; all samples when none fall in it."""
        if self.proc is None or not self.lines:
            return None
        t0, t1 = window if window is not None else (self.t0, self.t1)
        rows = []
        if t0 is not None:
            rows = [l for (t, l) in self.lines if t0 - 0.25 <= t <= (t1 or t) + 0.25]
        in_window = bool(rows)
        rows = rows or [l for _, l in self.lines]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            parts = [x.strip() for x in r.split(",")]
            if len(parts) < 10:
                continue
            try:
                sm.append(float(parts[2]))
                smax.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "in_window": in_window}


# ----------------------------------------------------------------- our arm

def decode_cfg(args):
    """The decode workload of --config, with --seq-len / --batch applied."""
    cfg = workloads.CONFIGS[args.config]
    over = {}
    if args.seq_len is not None:
        over["S"] = args.seq_len
    if args.batch is not None:
        over["B"] = args.batch
    return workloads.scaled(cfg.name, **over) if over else cfg


def workload_desc(c) -> str:
    if c.chunk_len:
        split = f"chunk_len={c.chunk_len}, S_b~U[{c.S_min},{c.S}]"
    else:
        split = f"S={c.S}, n_splits={c.n_splits}"
    return (f"{c.name}: B={c.B}, h_q={c.h_q}, h_kv={c.h_kv}, d_head={c.d}, {split}, "
            f"{c.dtype} q/k/v, fp32 out")


def tensor_sha256(t: torch.Tensor) -> str:
    """First 16 hex digits of the SHA-256 of a CPU tensor's bytes."""
    return hashlib.sha256(t.contiguous().view(-1).view(torch.uint8).numpy()).hexdigest()[:16]


def input_hashes(w) -> dict:
    return {name: tensor_sha256(getattr(w, name)) for name in ("q", "k", "v", "seqlens")}


def rotation_copies(kv_bytes: int) -> int:
    """K/V copies the timed steps rotate through: >= 1 GiB in total (so no
    step finds its K/V in the 126 MB L2), at most 4096 (the tiny workload)."""
    return max(1, min(4096, math.ceil(ROTATE_TOTAL / max(kv_bytes, 1))))


def l2_note(n_copies: int, kv_bytes: int) -> str:
    return (f"K/V rotate among {n_copies} copies ({n_copies * kv_bytes / 2**30:.2f} GiB); "
            f"each step's K/V ({kv_bytes / 2**20:.2f} MiB) "
            + ("exceeds" if kv_bytes > L2_BYTES else "is below") + " the 126 MB L2")


def decode_config(cfg, w, world: int, seed) -> dict:
    """The `config` object of a decode line; both arms print the same one."""
    n_copies = rotation_copies(w.kv_bytes)
    return {
        "workload": workload_desc(cfg),
        "seed": cfg.seed if seed is None else seed,
        "kv_bytes_per_step": w.kv_bytes,
        "global_batch": cfg.B * world,
        "seq_len": cfg.S,
        "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        "l2": l2_note(n_copies, w.kv_bytes),
        "sha256_q_k_v_seqlens": input_hashes(w),
    }


class DecodeRig:
    """One decode workload resident on the device: rotating K/V copies, the
    workspace, and the fused and partial + merge calls of step i."""

    def __init__(self, gk, cfg, w, device):
        self.gk, self.cfg, self.w, self.device = gk, cfg, w, device
        self.kv_bytes = w.kv_bytes
        self.n_copies = rotation_copies(self.kv_bytes)
        self.q = w.q.to(device)
        self.sl = w.seqlens.to(device)
        k0, v0 = w.k.to(device), w.v.to(device)
        self.ks, self.vs = [k0], [v0]
        if self.n_copies > 1:
            kk = torch.empty((self.n_copies - 1,) + tuple(k0.shape), dtype=k0.dtype, device=device)
            vv = torch.empty_like(kk)
            kk.copy_(k0.unsqueeze(0).expand_as(kk))
            vv.copy_(v0.unsqueeze(0).expand_as(vv))
            self.ks += list(kk.unbind(0))
            self.vs += list(vv.unbind(0))
        self.out = torch.empty((cfg.B, cfg.h_q, cfg.d), dtype=torch.float32, device=device)
        self.max_seqlen = w.max_seqlen
        if cfg.chunk_len:
            self.n_slots = max(1, -(-self.max_seqlen // cfg.chunk_len))
            ws = gk.chunked_workspace_size(cfg.B, cfg.h_q, cfg.h_kv, cfg.d, cfg.chunk_len, self.max_seqlen)
        else:
            self.n_slots = cfg.n_splits
            ws = gk.workspace_size(cfg.B, cfg.h_q, cfg.h_kv, cfg.d, cfg.n_splits)
        self.ws = torch.zeros(ws, dtype=torch.uint8, device=device)
        dt = gk.BF16 if cfg.dtype == "bf16" else gk.F32
        self.launches = gk.launches_per_call(cfg.B, cfg.h_q, cfg.h_kv, cfg.d, self.n_slots, dt, device)
        self.plan = gk.fused_plan(cfg.B, cfg.h_q, cfg.h_kv, cfg.d, self.n_slots, dt, device)
        shape = (cfg.B, cfg.h_q, self.n_slots)
        self.m = torch.empty(shape, dtype=torch.float32, device=device)
        self.l = torch.empty(shape, dtype=torch.float32, device=device)
        self.o = torch.empty(shape + (cfg.d,), dtype=torch.float32, device=device)

    def fused(self, i):
        c, j = self.cfg, i % self.n_copies
        if c.chunk_len:
            self.gk.gqa_decode_attn_chunked(self.q, self.ks[j], self.vs[j], self.sl, c.chunk_len,
                                            self.max_seqlen, c.scale, out=self.out, workspace=self.ws)
        else:
            self.gk.gqa_decode_attn(self.q, self.ks[j], self.vs[j], self.sl, c.n_splits, c.scale,
                                    out=self.out, workspace=self.ws)

    def partial_merge(self, i):
        c, j = self.cfg, i % self.n_copies
        if c.chunk_len:
            self.gk.gqa_decode_partial_chunked(self.q, self.ks[j], self.vs[j], self.sl, c.chunk_len,
                                               self.max_seqlen, c.scale, m=self.m, l=self.l, o=self.o)
        else:
            self.gk.gqa_decode_partial(self.q, self.ks[j], self.vs[j], self.sl, c.n_splits, c.scale,
                                       m=self.m, l=self.l, o=self.o)
        self.gk.mlo_merge(self.m, self.l, self.o, out=self.out)

    def kernel_name(self) -> str:
        if self.plan == "simt":
            return "decode_simt_f32 (fused, ticket merge)"
        if self.plan == "persistent":
            return "decode_tc_bf16_persist + merge_rows_kernel"
        if self.launches == 2:
            return f"decode_tc_bf16 ({self.plan}) + merge_rows_kernel"
        return f"decode_tc_bf16 ({self.plan}, ticket merge)"


def upload_graph(g, stream) -> bool:
    """Uploads an instantiated CUDA graph to the device ahead of its first
    replay (so the replay that is timed does not pay for it)."""
    try:
        try:
            from cuda.bindings import runtime as rt
        except ImportError:  # older cuda-python
            from cuda import cudart as rt
        err = rt.cudaGraphUpload(g.raw_cuda_graph_exec(), stream.cuda_stream)[0]
        return int(err) == 0
    except Exception:
        return False


# Device cycles of the stream hold queued before a device-timed region
# (about 0.1 ms at the B200's clocks).  torch.cuda._sleep is torch's own
# bounded spin kernel (a private helper): without it the regions start on an
# idle GPU, and the JSON line says so.
HOLD_CYCLES = 200_000
HOLD_AVAILABLE = hasattr(torch.cuda, "_sleep")


def hold_stream(stream):
    """Queues the bounded spin on `stream`; False when torch lacks it."""
    if not HOLD_AVAILABLE:
        return False
    with torch.cuda.stream(stream):
        torch.cuda._sleep(HOLD_CYCLES)
    return True


def _timed_region(run, device, world, hold: bool = False):
    """One timed region: barrier + synchronize, CUDA events on the launching
    stream around run(), synchronize + barrier.  Returns (device ms, host
    wall window).

    hold: queue a bounded spin (torch.cuda._sleep, HOLD_CYCLES) ahead of the
    start event, so the GPU is still busy with it while the host submits
    run()'s work; the region then starts when the first step does, not when
    the host's submission reaches an idle GPU (the blocking-kernel method of
    GPU benchmark harnesses).  Every step of run() stays inside the region."""
    stream = torch.cuda.current_stream(device)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(device)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0 = time.time()
    if hold:
        hold_stream(stream)
    s.record(stream)
    run()
    e.record(stream)
    torch.cuda.synchronize(device)
    h1 = time.time()
    if world > 1:
        dist.barrier()
    return s.elapsed_time(e), (h0, h1)


def decode_loop_e2e(gk, cfg, w, rig, E: int, device, world: int):
    """End to end as a decode loop runs: the KV cache stays resident in a
    padded layout ([B][S_max + 1][h_kv][d]); every step copies q and the new
    token's k and v in from pinned host memory, calls gqa_decode_attn_append
    (which writes the token into the cache and attends over S_b + 1 keys) and
    copies the result back.  seqlens is not advanced, so every step redoes
    the same work (the new row is rewritten in place)."""
    B, hkv, d = cfg.B, cfg.h_kv, cfg.d
    sl = w.seqlens.tolist()
    cap = max(sl) + 1
    kp = torch.zeros((B, cap, hkv, d), dtype=w.k.dtype, device=device)
    vp = torch.zeros_like(kp)
    off = 0
    for b, S in enumerate(sl):
        kp[b, :S].copy_(w.k[off:off + S])
        vp[b, :S].copy_(w.v[off:off + S])
        off += S
    gen = torch.Generator().manual_seed(cfg.seed + 7)
    # q and the new token's k, v side by side in one pinned buffer, so a step
    # moves its inputs with one host-to-device copy (views of one device buffer)
    nq, nkv = B * cfg.h_q * d, B * hkv * d
    hin = torch.empty(nq + 2 * nkv, dtype=w.q.dtype).pin_memory()
    hin[:nq].copy_(w.q.reshape(-1))
    hin[nq:].copy_(torch.randn(2 * nkv, generator=gen).to(w.q.dtype))
    din = torch.empty_like(hin, device=device)
    dq = din[:nq].view(B, cfg.h_q, d)
    dkn = din[nq:nq + nkv].view(B, hkv, d)
    dvn = din[nq + nkv:].view(B, hkv, d)
    hout = torch.empty((B, cfg.h_q, d), dtype=torch.float32).pin_memory()
    dsl = w.seqlens.to(device)
    ws = torch.zeros(gk.workspace_size(B, cfg.h_q, hkv, d, cfg.n_splits), dtype=torch.uint8, device=device)
    out = torch.empty((B, cfg.h_q, d), dtype=torch.float32, device=device)

    def step():
        din.copy_(hin, non_blocking=True)
        gk.gqa_decode_attn_append(dq, dkn, dvn, kp, vp, dsl, cfg.n_splits, cfg.scale, out=out, workspace=ws)
        hout.copy_(out, non_blocking=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize(device)
    ms, _ = _timed_region(lambda: [step() for _ in range(E)], device, world)
    check_status(gk, device, "after the decode-loop end-to-end steps")
    ms = max_over_ranks(ms / E, world, device)
    kv = 2 * sum(S + 1 for S in sl) * hkv * d * w.k.element_size()
    total = sum_over_ranks(float(kv), world, device)
    del kp, vp, ws
    return {
        "value": round(total / (ms * 1e-3) / 1e9, 2),
        "unit": UNIT,
        "h2d_bytes_per_step": hin.numel() * hin.element_size(),
        "d2h_bytes_per_step": hout.numel() * hout.element_size(),
        "ms_per_step": round(ms, 5),
        "kv_bytes_per_step": kv,
        "note": "decode-loop form: the cache resident on the GPU (padded, S_max + 1 rows); q and the new "
                "token's k, v copied in from one pinned buffer, gqa_decode_attn_append (append + attend over "
                "S_b + 1 keys), the result copied back; direct calls, every step",
    }


def timed_steps(call, K: int, W: int, device, world: int, graph: bool = True, hold: bool = True):
    """W untimed warm-up steps, then exactly K steps timed twice: as K direct
    calls of the public API, and (graph=True) as one replay of a CUDA graph of
    those same K calls, captured and uploaded before its timed region -- every
    step's kernels run unchanged; only the host's launch work leaves the
    timed region.  hold: see _timed_region.  Returns (direct ms, graph ms or
    None, the graph's host window or the direct one)."""
    stream = torch.cuda.current_stream(device)
    for i in range(W):
        call(i)
    torch.cuda.synchronize(device)
    direct_ms, win = _timed_region(lambda: [call(W + i) for i in range(K)], device, world, hold)
    if not graph:
        return direct_ms, None, win
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    # thread-local capture: CUDA calls of other host threads (a process
    # group's watchdog) neither join nor break the capture
    with torch.cuda.graph(g, stream=side, capture_error_mode="thread_local"):
        for i in range(K):
            call(W + i)
    stream.wait_stream(side)
    upload_graph(g, stream)
    torch.cuda.synchronize(device)
    graph_ms, win = _timed_region(g.replay, device, world, hold)
    del g
    return direct_ms, graph_ms, win


def check_status(gk, device, where: str):
    status = gk.get_status(device)
    if status != 0:
        raise RuntimeError(f"device status {status} {where}")


def per_config_entry(gk, name, args, device, sampler, peak):
    """One more decode workload timed like the headline (same steps and
    warm-up), on one GPU."""
    cfg = workloads.CONFIGS[name]
    w = workloads.generate(cfg, seed=args.seed)
    rig = DecodeRig(gk, cfg, w, device)
    direct_ms, graph_ms, win = timed_steps(rig.fused, args.steps, args.warmup, device, 1,
                                           graph=not args.no_graph, hold=not args.no_hold)
    check_status(gk, device, f"after timing {name}")
    us = (graph_ms if graph_ms is not None else direct_ms) * 1e3 / args.steps
    us_direct = direct_ms * 1e3 / args.steps
    gbs = rig.kv_bytes / (us * 1e-6) / 1e9
    entry = {
        "workload": workload_desc(cfg),
        "us_per_call": round(us, 3),
        "value_gbs": round(gbs, 2),
        "frac_of_hbm_peak": round(gbs / peak, 4),
        "timing": ("CUDA graph of the K calls" if graph_ms is not None else "direct calls")
                  + ("" if args.no_hold or not HOLD_AVAILABLE else ", device spin queued ahead of the start event"),
        "direct_calls_us_per_call": round(us_direct, 3),
        "direct_calls_frac_of_hbm_peak": round(rig.kv_bytes / (us_direct * 1e-6) / 1e9 / peak, 4),
        "kv_bytes_per_step": rig.kv_bytes,
        "steps": args.steps,
        "warmup": args.warmup,
        "kernel": rig.kernel_name(),
        "launches_per_step": rig.launches,
        "l2": l2_note(rig.n_copies, rig.kv_bytes),
        "sha256_q_k_v_seqlens": input_hashes(w),
        "clocks": sampler.summary(win),
    }
    out = rig.out.detach().cpu()   # the output of the last timed step
    del rig, w
    torch.cuda.empty_cache()
    return entry, out


def run_ours(args, rank, world, local_rank):
    import gqa_split_kv_decode_b200 as gk

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    # The clock sampler runs from before the first warm-up step, so the timed
    # steps follow the warm-up directly (no idle gap before the timed region).
    sampler = ClockSampler(device.index if device.index is not None else 0)
    if rank == 0 and not args.no_clocks:
        sampler.start()
    cfg = decode_cfg(args)
    w = workloads.generate(cfg, seed=args.seed)
    kv_bytes = w.kv_bytes
    rig = DecodeRig(gk, cfg, w, device)
    stream = torch.cuda.current_stream(device)

    K = args.steps
    direct_ms, graph_ms, win = timed_steps(rig.fused, K, args.warmup, device, world,
                                           graph=not args.no_graph, hold=not args.no_hold)
    total_ms = graph_ms if graph_ms is not None else direct_ms
    check_status(gk, device, "after the timed region")
    out_host = rig.out.detach().cpu()   # the output of the last timed step
    clocks = sampler.summary(win) if rank == 0 else None
    max_direct_ms = max_over_ranks(direct_ms, world, device)

    # one launch at a time (events around each call; no overlap between calls)
    n_iso = min(K, 200)
    iso_s = [torch.cuda.Event(enable_timing=True) for _ in range(n_iso)]
    iso_e = [torch.cuda.Event(enable_timing=True) for _ in range(n_iso)]
    for i in range(n_iso):
        iso_s[i].record(stream)
        rig.fused(i)
        iso_e[i].record(stream)
    torch.cuda.synchronize(device)
    iso_all = [a.elapsed_time(b) for a, b in zip(iso_s, iso_e)]
    iso_ms = float(np.median(iso_all))
    iso_p10, iso_p90 = (max_over_ranks(float(np.percentile(iso_all, q)), world, device) for q in (10, 90))

    # the same workload through the two-call form: gqa_decode_partial + mlo_merge
    pm_direct, pm_graph, _ = timed_steps(rig.partial_merge, K, args.warmup, device, world,
                                         graph=not args.no_graph, hold=not args.no_hold)
    check_status(gk, device, "after timing partial + merge")
    max_pm_ms = max_over_ranks(pm_graph if pm_graph is not None else pm_direct, world, device)

    max_total_ms = max_over_ranks(total_ms, world, device)
    max_iso_ms = max_over_ranks(iso_ms, world, device)
    all_bytes = sum_over_ranks(float(kv_bytes) * K, world, device)

    # ---- end to end through the public API: pinned host inputs in, result out
    E = max(1, min(args.e2e_steps, K))
    hq = w.q.pin_memory()
    hk = w.k.pin_memory()
    hv = w.v.pin_memory()
    hsl = w.seqlens.pin_memory()
    hout = torch.empty_like(rig.out, device="cpu").pin_memory()
    dq, dk, dv, dsl = (torch.empty_like(t, device=device) for t in (w.q, w.k, w.v, w.seqlens))

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        dsl.copy_(hsl, non_blocking=True)
        if cfg.chunk_len:
            gk.gqa_decode_attn_chunked(dq, dk, dv, dsl, cfg.chunk_len, w.max_seqlen, cfg.scale,
                                       out=rig.out, workspace=rig.ws)
        else:
            gk.gqa_decode_attn(dq, dk, dv, dsl, cfg.n_splits, cfg.scale, out=rig.out, workspace=rig.ws)
        hout.copy_(rig.out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / E, world, device)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hsl))
    d2h = hout.numel() * hout.element_size()
    e2e_bytes = sum_over_ranks(float(kv_bytes), world, device)
    loop = decode_loop_e2e(gk, cfg, w, rig, E, device, world) if not cfg.chunk_len else None
    launches = rig.launches
    kernel = rig.kernel_name()
    del rig, dq, dk, dv, dsl
    torch.cuda.empty_cache()

    peak, peak_src = measured_hbm_peak()
    per_config = None
    gpu_outs = {cfg.name: out_host}
    if world == 1 and not args.no_per_config and cfg == workloads.CONFIGS.get(cfg.name):
        per_config = {}
        for name in workloads.CONFIGS:
            if name != cfg.name:
                per_config[name], gpu_outs[name] = per_config_entry(gk, name, args, device, sampler, peak)
    sampler.stop()

    if rank != 0:
        return None

    ms_per_step = max_total_ms / K
    value = all_bytes / (max_total_ms * 1e-3) / 1e9
    achieved = kv_bytes / (ms_per_step * 1e-3) / 1e9
    traffic = profiled_traffic(cfg.name) if cfg == workloads.CONFIGS.get(cfg.name) else None
    pm_us = max_pm_ms * 1e3 / K
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 6),
        "us_per_call": round(ms_per_step * 1e3, 3),
        "pct_of_hbm_peak": round(100.0 * value / (peak * world), 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v; no dataset or weights involved)",
        "config": decode_config(cfg, w, world, args.seed),
        "accumulate": "fp32 (bf16 tensor-core products, fp32 softmax and merge)",
        "roofline": {
            "bound": "hbm",
            "achieved": round(achieved, 2),
            "peak": peak,
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, copy)" if peak_src == "measured" else "fallback",
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": traffic,
            "traffic_source": ("dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture, read from the "
                               "committed summary profiles/decode_tc_bf16_persist_llama70b.md (taken on the "
                               "current kernel sources: their hash matches), not measured in this run")
                              if traffic is not None else "none: no ncu summary of the current kernel sources",
            "algorithmic_bytes_per_launch": kv_bytes,
            "kernel": kernel,
            "launches_per_step": launches,
            "timing": ("CUDA events around one replay of a CUDA graph of the K public-API calls, captured "
                       "and uploaded before the timed region (every step's kernels unchanged; the host's "
                       "launch work out of the timed region); a step's launches together, so the dominant "
                       "kernel's own rate is at least this" if graph_ms is not None else
                       "CUDA events around the K back-to-back calls of the timed region (a step's launches "
                       "together, so the dominant kernel's own rate is at least this)")
                      + ("; a bounded device spin (torch.cuda._sleep) queued ahead of the start event keeps "
                         "the GPU busy while the host submits the steps, so the region starts with the first "
                         "step" if not args.no_hold and HOLD_AVAILABLE else "; the region starts on an idle GPU"),
            "launch_ms": round(ms_per_step, 6),
            "isolated_launch_ms": round(max_iso_ms, 6),
            "isolated_launch_ms_p10_p90": [round(iso_p10, 6), round(iso_p90, 6)],
        },
        "direct_calls": {
            "what": "the same K steps as K direct calls of the public API, host launch work inside the "
                    "timed region",
            "ms_per_step": round(max_direct_ms / K, 6),
            "value": round(all_bytes / (max_direct_ms * 1e-3) / 1e9, 2),
            "frac_of_hbm_peak": round(kv_bytes / (max_direct_ms / K * 1e-3) / 1e9 / peak, 4),
        },
        "partial_merge": {
            "what": "the same workload as gqa_decode_partial (triplets to HBM) + mlo_merge, two calls per step",
            "us_per_call": round(pm_us, 3),
            "value_gbs": round(kv_bytes / (pm_us * 1e-6) / 1e9, 2),
            "frac_of_hbm_peak": round(kv_bytes / (pm_us * 1e-6) / 1e9 / peak, 4),
            "steps": K,
            "warmup": args.warmup,
        },
        "e2e": {
            "value": round(e2e_bytes / (e2e_ms * 1e-3) / 1e9, 3),
            "unit": UNIT,
            "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "ms_per_step": round(e2e_ms, 4),
            "note": "pinned host q/k/v/seqlens (the whole cache) copied in and out copied back every step",
        },
        "gpu_launches": K * launches,
        "clocks": clocks,
    }
    if loop is not None:
        line["e2e_decode_loop"] = loop
    if per_config is not None:
        line["per_config"] = per_config
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=20.0, gpu_out=out_host)
        line["cpu_baseline"]["single_core"] = single_core_baselines(args.seed, gpu_outs=gpu_outs)
    return line


# ------------------------------------------------------- the CPU oracle arm

def oracle_sample(w, n_items: int, start: int):
    """n_items (b, h) pairs of the workload, cycling through all of them."""
    c = w.cfg
    total = c.B * c.h_q
    idx = [(start + i) % total for i in range(n_items)]
    return [(i // c.h_q, i % c.h_q) for i in idx]


def sample_parity(cfg, items, ref, gpu_out) -> dict:
    """The GPU output of the timed steps against the oracle rows computed for
    the CPU baseline: max abs error, max rel error over |ref| >= 0.2, and the
    worst error as a fraction of the elementwise bound atol + rtol |ref|."""
    atol, rtol = (2e-3, 1e-2) if cfg.dtype == "bf16" else (1e-5, 1e-5)
    got = np.stack([gpu_out[b, h].double().numpy() for b, h in items])
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    big = np.abs(ref) >= 0.2
    worst = float((err / (atol + rtol * np.abs(ref))).max())
    return {"rows": len(items), "max_abs_err": float(err.max()),
            "max_rel_err": float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0,
            "worst_err_over_bound": round(worst, 5), "bound": f"{atol:g} + {rtol:g}*|ref|",
            "pass": bool(worst <= 1.0)}


def cpu_baseline(w, budget_s: float, gpu_out=None):
    """Times the oracle as it stands on a sample of (b, h) rows; KV GB/s is
    the workload's KV bytes scaled by the sampled fraction of its rows.  The
    rows of the first pass also check the GPU output of the timed steps
    (`gpu_out`, host copy) when it is given."""
    import oracle
    c = w.cfg
    total = c.B * c.h_q
    cores = os.cpu_count() or 1
    n = min(total, max(cores, 1))
    t0 = time.perf_counter()
    first = oracle_sample(w, n, 0)
    ref0 = oracle.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale, items=first)
    dt = time.perf_counter() - t0
    per_item = dt / n
    n_run = int(max(n, budget_s / max(per_item, 1e-9)))
    t0 = time.perf_counter()
    done, start = 0, n
    while done < n_run:
        m = min(total, n_run - done)
        oracle.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale, items=oracle_sample(w, m, start))
        start += m
        done += m
    dt = time.perf_counter() - t0
    kv_equiv = w.kv_bytes * done / total
    res = {"value": round(kv_equiv / dt / 1e9, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
           "sample": f"{done} (b, h) output rows, cycling through the workload's {total} "
                     f"({done / total:.2f} passes; fp64 two-pass, {dt:.1f} s); KV bytes "
                     f"scaled by the rows done",
           "seconds": round(dt, 2)}
    if gpu_out is not None:
        res["parity"] = sample_parity(c, first, ref0, gpu_out)
    return res


def single_core_baselines(seed, budget_s: float = 2.0, gpu_outs=None) -> dict:
    """The oracle on ONE host thread for the tiny, Llama-2-7B and Llama-70B
    workloads: (b, h) rows for about `budget_s` each, KV GB/s scaled by the
    rows done.  Rows computed here also check the GPU output of that
    workload's timed steps when `gpu_outs` holds it."""
    import oracle
    res = {}
    for name in ("tiny", "llama7b", "llama70b"):
        w = workloads.generate(workloads.CONFIGS[name], seed=seed)
        c = w.cfg
        total = c.B * c.h_q
        done, start, dt = 0, 0, 0.0
        items, refs = [], []
        while dt < budget_s and done < 64 * total:
            it = oracle_sample(w, 1, start)
            t0 = time.perf_counter()
            r = oracle.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale, items=it, nthreads=1)
            dt += time.perf_counter() - t0
            if done < total:
                items += it
                refs.append(r[0])
            start += 1
            done += 1
        res[name] = {"value": round(w.kv_bytes * done / total / dt / 1e9, 4), "unit": UNIT, "cores": 1,
                     "sample": f"{done} of {total} (b, h) rows, {dt:.2f} s"}
        if gpu_outs and name in gpu_outs:
            res[name]["parity"] = sample_parity(c, items, np.stack(refs), gpu_outs[name])
    return res


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    cfg = decode_cfg(args)
    w = workloads.generate(cfg, seed=args.seed)
    c = w.cfg
    total = c.B * c.h_q
    cores = os.cpu_count() or 1
    # size each step so the whole run stays near two minutes
    t0 = time.perf_counter()
    oracle.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale, items=oracle_sample(w, cores, 0))
    per_item = (time.perf_counter() - t0) / cores
    steps = args.steps + args.warmup
    n_items = int(max(1, min(total, 120.0 / max(steps, 1) / max(per_item, 1e-9))))
    for i in range(args.warmup):
        oracle.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale, items=oracle_sample(w, n_items, i * n_items))
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.attn(w.q, w.k, w.v, w.seqlens, c.h_q, c.h_kv, c.scale,
                    items=oracle_sample(w, n_items, (args.warmup + i) * n_items))
    dt = time.perf_counter() - t0
    kv_equiv = w.kv_bytes * n_items / total * args.steps
    value = kv_equiv / dt / 1e9
    sample = f"{n_items} of {total} (b, h) output rows per step; KV bytes scaled by that fraction"
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / max(1, args.steps), 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v; no dataset or weights involved)",
        "config": decode_config(cfg, w, world, args.seed),
        "accumulate": "fp64 (the CPU oracle: two-pass softmax, no splitting)",
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------- sharded decode arm

def run_sharded(args, rank, world, local_rank):
    import gqa_split_kv_decode_b200 as gk
    from gqa_split_kv_decode_b200 import sharded

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    cfg = decode_cfg(args)
    w = workloads.generate(cfg, seed=args.seed)
    k_loc, v_loc, sl_loc = sharded.shard_packed_cache(w.k, w.v, w.seqlens, rank, world)
    local_bytes = 2 * k_loc.numel() * k_loc.element_size()
    n_copies = max(1, math.ceil(ROTATE_TOTAL / max(local_bytes, 1)))
    q = w.q.to(device)
    sl = sl_loc.to(device)
    ks = [k_loc.to(device) for _ in range(n_copies)]
    vs = [v_loc.to(device) for _ in range(n_copies)]
    n = gk.auto_splits(cfg.B, cfg.h_q, cfg.h_kv, cfg.d, int(sl_loc.max()) if cfg.B else 0, device)
    out = torch.empty((cfg.B, cfg.h_q, cfg.d), dtype=torch.float32, device=device)

    def call(i):
        sharded.sharded_decode(q, ks[i % n_copies], vs[i % n_copies], sl, n, cfg.scale, out=out)

    sampler = ClockSampler(device.index if device.index is not None else 0)
    if rank == 0 and not args.no_clocks:
        sampler.start()
    for i in range(args.warmup):
        call(i)
    torch.cuda.synchronize(device)
    if gk.get_status(device) != 0:
        raise RuntimeError("device status set during warm-up")
    K = args.steps
    stream = torch.cuda.current_stream(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(device)
    sampler.mark_begin()
    if not args.no_hold:  # as in _timed_region
        hold_stream(stream)
    t0.record(stream)
    for i in range(K):
        call(i)
    t1.record(stream)
    torch.cuda.synchronize(device)
    sampler.mark_end()
    if world > 1:
        dist.barrier()
    total_ms = max_over_ranks(t0.elapsed_time(t1), world, device)
    if gk.get_status(device) != 0:
        raise RuntimeError("device status set in the timed region")
    sampler.stop()
    clocks = sampler.summary() if rank == 0 else None

    E = max(1, min(args.e2e_steps, K))
    hq, hk, hv, hsl = (t.pin_memory() for t in (w.q, k_loc, v_loc, sl_loc))
    hout = torch.empty_like(out, device="cpu").pin_memory()
    dk, dv = torch.empty_like(ks[0]), torch.empty_like(vs[0])

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        sl.copy_(hsl, non_blocking=True)
        sharded.sharded_decode(q, dk, dv, sl, n, cfg.scale, out=out)
        hout.copy_(out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / E, world, device)
    max_local = max_over_ranks(float(local_bytes), world, device)
    if rank != 0:
        return None
    peak, peak_src = measured_hbm_peak()
    ms = total_ms / K
    value = w.kv_bytes / (ms * 1e-3) / 1e9
    return {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms, 6), "us_per_call": round(ms * 1e3, 3),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v; no dataset or weights involved)",
        "config": {"workload": workload_desc(cfg), "kv_bytes_per_step": w.kv_bytes,
                   "seed": cfg.seed if args.seed is None else args.seed,
                   "global_batch": cfg.B, "seq_len": cfg.S,
                   "parallelism": f"sequence-sharded KV over {world} ranks, {n} splits per rank",
                   "l2": f"each rank's K/V shard rotates among {n_copies} copies"},
        "roofline": {"bound": "hbm", "achieved": round(max_local / (ms * 1e-3) / 1e9, 2), "peak": peak,
                     "peak_source": peak_src, "unit": "GB/s",
                     "frac": round(max_local / (ms * 1e-3) / 1e9 / peak, 4), "traffic": None,
                     "kernel": "decode_tc_bf16 (partial) + mlo_merge_ranked_kernel, NCCL all-gather between",
                     "note": "achieved = the largest rank's shard bytes / step time (all-gather included)"},
        "e2e": {"value": round(w.kv_bytes / (e2e_ms * 1e-3) / 1e9, 3), "unit": UNIT,
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (hq, hk, hv, hsl)),
                "d2h_bytes_per_step": hout.numel() * hout.element_size(), "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": 2 * K,
        "clocks": clocks,
    }


# ------------------------------------------------------------ prefill arm

def prefill_desc(w) -> str:
    sl = w.seqlens.tolist()
    lens = f"S={sl[0]}" if len(set(sl)) == 1 else f"S_b in [{min(sl)}, {max(sl)}] (seeded)"
    return (f"{w.name}: causal prefill, B={len(sl)}, {lens}, h_q={w.h_q}, h_kv={w.h_kv}, "
            f"d_head={w.d}, bf16 q/k/v, fp32 out")


def prefill_items(w, n: int, start: int):
    """n (b, h, i) output rows of the workload, spread over all of them."""
    sl = w.seqlens.tolist()
    off = np.concatenate([[0], np.cumsum(sl)])
    total = int(off[-1]) * w.h_q
    items = []
    for k in range(n):
        x = ((start + k) * 7919) % total        # a fixed stride walk over (row, head)
        row, h = divmod(x, w.h_q)
        b = int(np.searchsorted(off, row, side="right") - 1)
        items.append((b, h, int(row - off[b])))
    return items


def prefill_item_flops(w, items) -> float:
    return float(sum(4 * w.d * (i + 1) for _, _, i in items))


def prefill_cpu_baseline(w, budget_s: float):
    import oracle
    cores = os.cpu_count() or 1
    n = max(cores, 64)
    t0 = time.perf_counter()
    oracle.prefill(w.q, w.k, w.v, w.seqlens, w.h_q, w.h_kv, w.scale, items=prefill_items(w, n, 0))
    per_item = (time.perf_counter() - t0) / n
    n_run = int(max(n, budget_s / max(per_item, 1e-9)))
    items = prefill_items(w, n_run, n)
    t0 = time.perf_counter()
    oracle.prefill(w.q, w.k, w.v, w.seqlens, w.h_q, w.h_kv, w.scale, items=items)
    dt = time.perf_counter() - t0
    return {"value": round(prefill_item_flops(w, items) / dt / 1e12, 6), "unit": "TFLOP/s",
            "cores": cores, "kind": "oracle",
            "sample": f"{n_run} (sequence, head, position) output rows of the workload (fp64 two-pass, "
                      f"{dt:.1f} s); FLOPs = 4 d (i + 1) per row",
            "seconds": round(dt, 2)}


def run_prefill(args, rank, world, local_rank):
    import gqa_split_kv_decode_b200 as gk

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    w = workloads.generate_prefill(args.config, seed=args.seed)
    flops = w.flops
    one = sum(t.numel() * t.element_size() for t in (w.q, w.k, w.v)) + w.q.numel() * 4
    n_copies = max(1, math.ceil(ROTATE_TOTAL / one))
    qs = [w.q.to(device) for _ in range(n_copies)]
    ks = [w.k.to(device) for _ in range(n_copies)]
    vs = [w.v.to(device) for _ in range(n_copies)]
    outs = [torch.empty(w.q.shape, dtype=torch.float32, device=device) for _ in range(n_copies)]
    sl = w.seqlens.to(device)
    ms = w.max_seqlen

    def call(i):
        c = i % n_copies
        gk.gqa_prefill_attn(qs[c], ks[c], vs[c], sl, w.scale, max_seqlen=ms, out=outs[c])

    sampler = ClockSampler(device.index if device.index is not None else 0)
    if rank == 0 and not args.no_clocks:
        sampler.start()
    for i in range(args.warmup):
        call(i)
    torch.cuda.synchronize(device)
    if gk.get_status(device) != 0:
        raise RuntimeError("device status set during warm-up")
    K = args.steps
    stream = torch.cuda.current_stream(device)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(device)
    sampler.mark_begin()
    if not args.no_hold:  # as in _timed_region
        hold_stream(stream)
    t_start.record(stream)
    for i in range(K):
        call(i)
    t_end.record(stream)
    torch.cuda.synchronize(device)
    sampler.mark_end()
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    if gk.get_status(device) != 0:
        raise RuntimeError("device status set in the timed region")
    sampler.stop()
    clocks = sampler.summary() if rank == 0 else None
    n_iso = min(K, 100)
    iso = []
    for i in range(n_iso):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call(i)
        b.record(stream)
        iso.append((a, b))
    torch.cuda.synchronize(device)
    iso_all = [a.elapsed_time(b) for a, b in iso]
    iso_ms = max_over_ranks(float(np.median(iso_all)), world, device)
    iso_p10, iso_p90 = (max_over_ranks(float(np.percentile(iso_all, q)), world, device) for q in (10, 90))
    max_total_ms = max_over_ranks(total_ms, world, device)
    all_flops = sum_over_ranks(float(flops) * K, world, device)

    # end to end: pinned host q/k/v/seqlens in, fp32 result out, every step
    E = max(1, min(args.e2e_steps, K))
    hq, hk, hv, hsl = (t.pin_memory() for t in (w.q, w.k, w.v, w.seqlens))
    hout = torch.empty(w.q.shape, dtype=torch.float32).pin_memory()
    dq, dk, dv, dsl = (torch.empty_like(t, device=device) for t in (w.q, w.k, w.v, w.seqlens))

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        dsl.copy_(hsl, non_blocking=True)
        gk.gqa_prefill_attn(dq, dk, dv, dsl, w.scale, max_seqlen=ms, out=outs[0])
        hout.copy_(outs[0], non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / E, world, device)
    e2e_flops = sum_over_ranks(float(flops), world, device)
    if rank != 0:
        return None

    burst, sustained, src = measured_bf16_peak()
    ms_per_step = max_total_ms / K
    long_region = max_total_ms > 1000.0
    peak = sustained if long_region else burst
    value = all_flops / (max_total_ms * 1e-3) / 1e12
    achieved = flops / (ms_per_step * 1e-3) / 1e12
    line = {
        "metric": PREFILL_METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 6),
        "us_per_call": round(ms_per_step * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v; no dataset or weights involved)",
        "config": {
            "workload": prefill_desc(w),
            "seed": "default (2000 + index)" if args.seed is None else args.seed,
            "flops_per_step": flops,
            "flop_count": "4 * d_head * h_q * sum_b S_b (S_b + 1) / 2: QK^T and PV over the causal pairs only",
            "global_batch": len(w.seqlens) * world,
            "seq_len": ms,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": f"q/k/v/out rotate among {n_copies} copies ({n_copies * one / 2**30:.2f} GiB)",
            "accumulate": "fp32 (bf16 tensor-core products in TMEM, fp32 softmax)",
        },
        "roofline": {
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": peak,
            "peak_source": (f"{src} MEASURED_PEAKS.json bf16_tflops_sustained (timed region > 1 s)"
                            if long_region else f"{src} MEASURED_PEAKS.json bf16_tflops (burst)"),
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "frac_of_burst_peak": round(achieved / burst, 4),
            "traffic": profiled_traffic(args.config, PREFILL_PROFILE, PREFILL_SOURCES),
            "algorithmic_flops_per_launch": flops,
            "kernel": "prefill_tc_bf16",
            "launches_per_step": 1,
            "launch_ms": round(ms_per_step, 6),
            "isolated_launch_ms": round(iso_ms, 6),
            "isolated_launch_ms_p10_p90": [round(iso_p10, 6), round(iso_p90, 6)],
        },
        "e2e": {
            "value": round(e2e_flops / (e2e_ms * 1e-3) / 1e12, 4),
            "unit": "TFLOP/s",
            "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (hq, hk, hv, hsl)),
            "d2h_bytes_per_step": hout.numel() * hout.element_size(),
            "ms_per_step": round(e2e_ms, 4),
            "note": "pinned host q/k/v/seqlens copied in and the fp32 output copied back every step",
        },
        "gpu_launches": K,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = prefill_cpu_baseline(w, budget_s=30.0)
    return line


def run_prefill_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    w = workloads.generate_prefill(args.config, seed=args.seed)
    cores = os.cpu_count() or 1
    t0 = time.perf_counter()
    oracle.prefill(w.q, w.k, w.v, w.seqlens, w.h_q, w.h_kv, w.scale, items=prefill_items(w, cores, 0))
    per_item = (time.perf_counter() - t0) / cores
    steps = args.steps + args.warmup
    n = int(max(1, 120.0 / max(steps, 1) / max(per_item, 1e-9)))
    for i in range(args.warmup):
        oracle.prefill(w.q, w.k, w.v, w.seqlens, w.h_q, w.h_kv, w.scale, items=prefill_items(w, n, i * n))
    flops = 0.0
    t0 = time.perf_counter()
    for i in range(args.steps):
        items = prefill_items(w, n, (args.warmup + i) * n)
        oracle.prefill(w.q, w.k, w.v, w.seqlens, w.h_q, w.h_kv, w.scale, items=items)
        flops += prefill_item_flops(w, items)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    sample = f"{n} (sequence, head, position) output rows per step; FLOPs = 4 d (i + 1) per row"
    return {
        "impl": "reference", "metric": PREFILL_METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3 / max(1, args.steps), 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, same workload as the GPU arm)",
        "config": {"workload": prefill_desc(w), "flops_per_step": w.flops,
                   "seed": "default (2000 + index)" if args.seed is None else args.seed},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    rank, world, local_rank = dist_env()
    if world != args.gpus and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    prefill = args.config in workloads.PREFILL_CONFIGS
    if args.impl == "reference":
        line = (run_prefill_reference if prefill else run_reference)(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        arm = run_prefill if prefill else (run_sharded if args.sharded else run_ours)
        line = arm(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
