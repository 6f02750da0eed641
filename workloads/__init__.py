"""Seeded synthetic decode workloads.

This module only draws numbers: it holds no attention arithmetic, and both the
oracle tests and the CUDA parity tests / benchmark take their inputs from it.

Shapes follow the pages: Llama-2 7B is multi-head (32 heads of 128), Llama-2
70B is grouped-query with 64 query heads over 8 kv heads of 128 (exllama
"Llama 2 is out", the 70B config.json), context 4096 for Llama-2.  Layout:

    q        [B, h_q, d]            one decode token per sequence
    k, v     [sum_b S_b, h_kv, d]   packed ragged cache, sequence b occupies
                                    rows S_0 + ... + S_{b-1} onwards
    seqlens  int32 [B]

Recipe (seed = 1000 + config index):
    1. seqlens (ragged config only): integers uniform in [128, 32768], from
       numpy PCG64(seed) -- the "main" generator of the later steps too;
    2. q, then k, then v: standard normals in fp32, times the config's std,
       rounded once to the storage dtype (bf16 round-to-nearest-even via
       torch).  Each tensor is drawn in chunks of 2**24 values; chunk c of
       tensor t (q = 0, k = 1, v = 2) comes from its own PCG64 seeded with
       SeedSequence([seed, t, c]), so the chunks are drawn in parallel and the
       values do not depend on the thread count;
    3. structure (from the main generator, in this order):
       - "llama70b": per sequence, round(0.001 * S) distinct key positions;
         for each kv head g, the minimum-norm vector delta with
         Q_g delta = (6 / scale) * 1 (Q_g = the group's bf16 queries) is added
         to k at those positions, so every query head of the group sees its
         logit raised by 6 (up to bf16 rounding of the result);
       - "ragged": each (row, kv head) v vector is multiplied by 10 with
         probability 0.01 (Bernoulli draws in row-major order), then rounded.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np
import torch

CHUNK = 1 << 24


@dataclass(frozen=True)
class Config:
    name: str
    index: int
    B: int
    h_q: int
    h_kv: int
    d: int
    S: int                    # keys per sequence (upper bound for ragged)
    dtype: str                # "f32" or "bf16"
    scale: float
    n_splits: int = 0         # split-count policy (0 = chunked)
    chunk_len: int = 0        # chunk policy (ragged)
    std: float = 1.0
    S_min: int = 0            # ragged lower bound (0 = uniform lengths)
    bias_frac: float = 0.0    # fraction of key positions given a logit bias
    bias: float = 0.0
    vscale_p: float = 0.0     # probability that a v row is scaled
    vscale: float = 1.0
    note: str = field(default="", compare=False)

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv


CONFIGS = {
    c.name: c
    for c in [
        Config("tiny", 1, B=1, h_q=4, h_kv=1, d=64, S=256, dtype="f32", scale=1 / math.sqrt(64),
               n_splits=4, note="fp32, N(0,1)"),
        Config("llama7b", 2, B=1, h_q=32, h_kv=32, d=128, S=4096, dtype="bf16",
               scale=1 / math.sqrt(128), n_splits=8, note="Llama-2-7B MHA, N(0,1)"),
        Config("llama70b", 3, B=8, h_q=64, h_kv=8, d=128, S=8192, dtype="bf16",
               scale=1 / math.sqrt(128), n_splits=8, bias_frac=0.001, bias=6.0,
               note="Llama-70B GQA, N(0,1), +6 logit bias on 0.1% of positions"),
        Config("longctx", 4, B=1, h_q=64, h_kv=8, d=128, S=1 << 20, dtype="bf16",
               scale=1 / math.sqrt(128), n_splits=64, std=0.5, note="1M keys, N(0,1)/2"),
        Config("ragged", 5, B=64, h_q=32, h_kv=8, d=128, S=32768, S_min=128, dtype="bf16",
               scale=1 / math.sqrt(128), chunk_len=1024, vscale_p=0.01, vscale=10.0,
               note="S_b ~ U[128, 32768], chunk 1024, 1% of v rows x10"),
    ]
}


@dataclass
class Workload:
    cfg: Config
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    seqlens: torch.Tensor

    @property
    def kv_bytes(self) -> int:
        """Bytes of K and V the method must read: every cached row once."""
        return 2 * int(self.seqlens.sum()) * self.cfg.h_kv * self.cfg.d * self.k.element_size()

    @property
    def max_seqlen(self) -> int:
        return int(self.seqlens.max()) if self.seqlens.numel() else 0


def _torch_dtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _normal(seed: int, tensor_id: int, shape, std: float, dtype) -> torch.Tensor:
    """Standard normals x std stored in ``dtype``; chunk c of the flat tensor
    is drawn from PCG64(SeedSequence([seed, tensor_id, c])), chunks in
    parallel threads (numpy and torch release the GIL while filling)."""
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(-1)
    n = flat.numel()

    def fill(c: int) -> None:
        s, e = c * CHUNK, min(n, (c + 1) * CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id, c])))
        x = g.standard_normal(e - s, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        flat[s:e] = torch.from_numpy(x).to(dtype)

    n_chunks = (n + CHUNK - 1) // CHUNK
    if n_chunks <= 1:
        for c in range(n_chunks):
            fill(c)
    else:
        with ThreadPoolExecutor(max_workers=min(n_chunks, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(n_chunks)))
    return out


def generate(cfg: Config, seed: int | None = None, seqlens=None) -> Workload:
    """Build the seeded inputs of ``cfg`` (see the module docstring)."""
    seed = cfg.seed if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    if seqlens is not None:
        sl = torch.as_tensor(np.asarray(seqlens, dtype=np.int32))
    elif cfg.S_min > 0:
        sl = torch.from_numpy(rng.integers(cfg.S_min, cfg.S, size=cfg.B, endpoint=True).astype(np.int32))
    else:
        sl = torch.full((cfg.B,), cfg.S, dtype=torch.int32)
    dt = _torch_dtype(cfg.dtype)
    rows = int(sl.sum())
    q = _normal(seed, 0, (cfg.B, cfg.h_q, cfg.d), cfg.std, dt)
    k = _normal(seed, 1, (rows, cfg.h_kv, cfg.d), cfg.std, dt)
    v = _normal(seed, 2, (rows, cfg.h_kv, cfg.d), cfg.std, dt)

    if cfg.bias_frac > 0.0:
        off = 0
        G = cfg.group
        for b in range(cfg.B):
            S = int(sl[b])
            n_pos = int(round(cfg.bias_frac * S))
            if n_pos > 0:
                pos = np.sort(rng.choice(S, size=n_pos, replace=False)) + off
                pos_t = torch.from_numpy(pos.astype(np.int64))
                for g in range(cfg.h_kv):
                    Qg = q[b, g * G:(g + 1) * G, :].double()
                    target = torch.full((G, 1), cfg.bias / cfg.scale, dtype=torch.float64)
                    delta = Qg.T @ torch.linalg.solve(Qg @ Qg.T, target)
                    rows_k = k[pos_t, g, :].double() + delta[:, 0]
                    k[pos_t, g, :] = rows_k.to(dt)
            off += S

    if cfg.vscale_p > 0.0:
        off = 0
        mask_rows = []
        for s in range(0, rows, CHUNK // max(1, cfg.h_kv)):
            e = min(rows, s + CHUNK // max(1, cfg.h_kv))
            m = rng.random((e - s, cfg.h_kv)) < cfg.vscale_p
            mask_rows.append(torch.from_numpy(m))
        mask = torch.cat(mask_rows) if mask_rows else torch.zeros((0, cfg.h_kv), dtype=torch.bool)
        idx = mask.nonzero(as_tuple=True)
        v[idx] = (v[idx].float() * cfg.vscale).to(dt)

    return Workload(cfg, q.contiguous(), k.contiguous(), v.contiguous(), sl.contiguous())


def scaled(name: str, **overrides) -> Config:
    """A config of the same structure with some sizes changed (test cases)."""
    return replace(CONFIGS[name], **overrides)


def random_case(B, h_q, h_kv, d, seqlens, dtype="bf16", seed=0, std=1.0, scale=None,
                n_splits=0, chunk_len=0) -> Workload:
    """A plain N(0, std^2) case with explicit sequence lengths (edge cases)."""
    cfg = Config("case", 0, B=B, h_q=h_q, h_kv=h_kv, d=d, S=max(list(seqlens) + [0]), dtype=dtype,
                 scale=(1 / math.sqrt(d)) if scale is None else scale, n_splits=n_splits,
                 chunk_len=chunk_len, std=std)
    return generate(cfg, seed=seed, seqlens=list(seqlens))


# ---------------------------------------------------------------- prefill

@dataclass
class PrefillWorkload:
    """Causal prefill inputs: q [rows, h_q, d], k, v [rows, h_kv, d], packed by
    sequence (sequence b occupies rows S_0 + ... + S_{b-1} onwards)."""
    name: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    seqlens: torch.Tensor
    h_q: int
    h_kv: int
    d: int
    scale: float

    @property
    def max_seqlen(self) -> int:
        return int(self.seqlens.max()) if self.seqlens.numel() else 0

    @property
    def flops(self) -> int:
        """Multiply-adds x 2 of the attended (query, key) pairs only: QK^T and
        PV, each 2 * d per pair per query head; pairs = S_b (S_b + 1) / 2."""
        pairs = sum(int(s) * (int(s) + 1) // 2 for s in self.seqlens.tolist())
        return 4 * self.d * self.h_q * pairs


# Llama-2 70B attention shape (64 query / 8 kv heads of 128) at the 2k
# prefill length of the tt-metal "[Llama2] Perf burndown" page; a ragged
# batch of the same shape.  Seeds 2000 + index.
PREFILL_CONFIGS = {
    "llama70b_prefill2k": dict(index=1, B=1, S=2048, S_min=0, h_q=64, h_kv=8, d=128),
    "prefill_ragged": dict(index=2, B=16, S=4096, S_min=1, h_q=64, h_kv=8, d=128),
}


def prefill_case(seqlens, h_q, h_kv, d, dtype="bf16", seed=0, std=1.0, scale=None,
                 name="case") -> PrefillWorkload:
    """N(0, std^2) causal-prefill inputs with explicit lengths: q, k, v drawn
    like the decode tensors (fp32 chunks from PCG64(SeedSequence([seed,
    tensor, chunk])), rounded once to ``dtype``)."""
    sl = torch.as_tensor(np.asarray(list(seqlens), dtype=np.int32))
    rows = int(sl.sum())
    dt = _torch_dtype(dtype)
    q = _normal(seed, 0, (rows, h_q, d), std, dt)
    k = _normal(seed, 1, (rows, h_kv, d), std, dt)
    v = _normal(seed, 2, (rows, h_kv, d), std, dt)
    return PrefillWorkload(name, q, k, v, sl, h_q, h_kv, d,
                           (1 / math.sqrt(d)) if scale is None else float(scale))


def generate_prefill(name: str, seed: int | None = None) -> PrefillWorkload:
    """The seeded prefill workload ``name``: lengths (ragged: uniform integers
    in [S_min, S] drawn first from seed 2000 + index, or ``seed``), then q,
    k, v."""
    c = PREFILL_CONFIGS[name]
    seed = 2000 + c["index"] if seed is None else seed
    if c["S_min"] > 0:
        rng = np.random.Generator(np.random.PCG64(seed))
        sl = rng.integers(c["S_min"], c["S"], size=c["B"], endpoint=True).tolist()
        seed += 100
    else:
        sl = [c["S"]] * c["B"]
    return prefill_case(sl, c["h_q"], c["h_kv"], c["d"], seed=seed, name=name)
