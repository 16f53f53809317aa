"""Seeded synthetic inputs for the block-sparse GQA attention workloads.

This module only draws numbers. It holds none of the arithmetic of the method
(no pooling, scoring, selection or attention), so that the CPU oracle and the
CUDA library can both be fed from it without sharing any of the computation
they are compared on.

Determinism across devices
--------------------------
Every large tensor is produced element by element from a counter-based hash
(two rounds of a 32-bit xor-shift-multiply mixer over the element's 64-bit
index), mapped through a fixed table of 2^20 standard-normal quantiles. All of
it is integer arithmetic plus IEEE single-rounded fp32 multiplies and adds done
as separate elementwise ops, so the same call gives the same bits on the CPU
and on a GPU, and any slice (one sequence, a range of positions) can be
regenerated on its own. Small parameters (planting directions, planted block
lists, page permutations, sequence lengths) are always computed on the CPU and
then copied.

Workloads
---------
The five workloads follow the problem statements of the pages (page 1,
"Summarizing the Breakthrough": per-query top-k over key blocks, GQA-shared
selection, a block cache used in prefill and decode; page 5: per-GQA-group
top-k over KV blocks at long context). Their sizes, value distributions and
planted "relevant blocks" are the synthetic stand-ins for long-context
retrieval workloads ("needles"): N(0,1) values, plus blocks whose keys are
shifted along a per-(sequence, KV group) unit direction u that is also added to
the queries, so that those blocks score far above the rest.
"""
from __future__ import annotations

import dataclasses
import math
from functools import lru_cache
from typing import Dict, List, Optional, Tuple

import torch

SEED_BASE = 0x5EED0000
_M32 = 0xFFFFFFFF
_TABLE_BITS = 20
_CHUNK = 1 << 25


# --------------------------------------------------------------------------
# counter-based normal generator
# --------------------------------------------------------------------------
@lru_cache(maxsize=None)
def _normal_table_cpu() -> torch.Tensor:
    """2^20 standard-normal quantiles at the cell midpoints, fp32."""
    n = 1 << _TABLE_BITS
    p = (torch.arange(n, dtype=torch.float64) + 0.5) / n
    return torch.special.ndtri(p).to(torch.float32)


_table_dev: Dict[str, torch.Tensor] = {}


def _normal_table(device: torch.device) -> torch.Tensor:
    key = str(device)
    if key not in _table_dev:
        _table_dev[key] = _normal_table_cpu().to(device)
    return _table_dev[key]


def _mix32(x: torch.Tensor) -> torch.Tensor:
    # x holds values in [0, 2^32) in int64; multipliers are < 2^31 so every
    # product stays below 2^63 (no signed overflow on any device).
    x = x ^ (x >> 16)
    x = (x * 0x7FEB352D) & _M32
    x = x ^ (x >> 15)
    x = (x * 0x2C1B3C6D) & _M32
    x = x ^ (x >> 16)
    return x


def _stream_key(*parts: int) -> Tuple[int, int]:
    """Two 32-bit keys from a tuple of small integers (CPU, pure Python)."""
    h1, h2 = 0x243F6A88, 0x85A308D3
    for p in parts:
        p &= (1 << 64) - 1
        for half in (p & _M32, p >> 32):
            h1 = (h1 ^ half) * 0x01000193 & _M32
            h1 ^= h1 >> 13
            h2 = (h2 + half * 0x9E3779B1) & _M32
            h2 = (h2 ^ (h2 >> 15)) * 0x2C1B3C6D & _M32
    return h1, h2


def gauss(key: Tuple[int, ...], start: int, count: int, device) -> torch.Tensor:
    """`count` fp32 N(0,1) draws for element indices start .. start+count-1."""
    device = torch.device(device)
    k1, k2 = _stream_key(*key)
    table = _normal_table(device)
    out = torch.empty(count, dtype=torch.float32, device=device)
    for c0 in range(0, count, _CHUNK):
        c1 = min(count, c0 + _CHUNK)
        n = torch.arange(start + c0, start + c1, dtype=torch.int64, device=device)
        lo = n & _M32
        hi = n >> 32
        h = _mix32(lo ^ k1)
        h = _mix32(h ^ ((hi + k2) & _M32))
        out[c0:c1] = table[h >> (32 - _TABLE_BITS)]
    return out


def uniform01(key: Tuple[int, ...], count: int) -> torch.Tensor:
    """`count` float64 uniforms in (0,1) on the CPU, from the same hash."""
    k1, k2 = _stream_key(*key)
    n = torch.arange(count, dtype=torch.int64)
    h = _mix32(_mix32(n ^ k1) ^ k2)
    return (h.to(torch.float64) + 0.5) / 4294967296.0


def cpu_generator(*key: int) -> torch.Generator:
    k1, k2 = _stream_key(*key)
    g = torch.Generator()
    g.manual_seed((k1 << 32) | k2)
    return g


# --------------------------------------------------------------------------
# workload definitions
# --------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    dtype: str           # "bf16" or "f32"
    batch: int
    hq: int
    hkv: int
    d: int
    block: int           # block size == page size
    top_k: int
    ctx: Tuple[int, ...]  # prefill: tokens per sequence; decode: cached tokens
    steps: int = 1       # decode steps (each appends one token, then attends)
    seed: int = SEED_BASE
    sigma_q: float = 1.0  # query noise scale
    a_q: float = 1.0      # query planting amplitude along u
    delta: float = 0.0    # key shift of planted blocks along u
    planted: Tuple[int, int] = (0, 0)  # planted block count drawn in [lo, hi]
    planted_region: float = 1.0  # planted blocks lie in the first fraction of ctx
    tiny_q_hat: bool = False     # tiny workload: plant along the last query's mean direction

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def total_len(self, b: int) -> int:
        """Tokens of sequence b once every step has appended its token."""
        return self.ctx[b] + (self.steps if self.kind == "decode" else 0)


def tiny_f32(**over) -> Workload:
    """batch 1, 1024 tokens, 1 KV / 4 query heads, d 64, block 64, top-k 4, fp32,
    with 2 planted blocks shifted by 0.5 along the last query's mean direction."""
    w = Workload(name="tiny_f32", kind="prefill", dtype="f32", batch=1, hq=4, hkv=1,
                 d=64, block=64, top_k=4, ctx=(1024,), seed=SEED_BASE + 0,
                 sigma_q=1.0, a_q=0.0, delta=0.5, planted=(2, 2),
                 planted_region=15 / 16, tiny_q_hat=True)
    return dataclasses.replace(w, **over)


def prefill_bf16(**over) -> Workload:
    """batch 1, 32768 tokens, 32 query / 4 KV heads, d 128, block 128, top-k 16, causal,
    q = 0.1 z + 0.25 u, 8 planted blocks per group with keys + 1.5 u."""
    w = Workload(name="prefill_bf16", kind="prefill", dtype="bf16", batch=1, hq=32, hkv=4,
                 d=128, block=128, top_k=16, ctx=(32768,), seed=SEED_BASE + 1,
                 sigma_q=0.1, a_q=0.25, delta=1.5, planted=(8, 8))
    return dataclasses.replace(w, **over)


def paged_decode_bf16(**over) -> Workload:
    """batch 32, 131072 cached tokens each, page = block = 64, 32 query / 8 KV heads,
    d 128, top-k 32, one appended token per sequence; q = z + u, 16 planted blocks
    per (sequence, group) with keys + 6 u."""
    batch = over.pop("batch", 32)
    ctx = over.pop("ctx", (131072,) * batch)
    w = Workload(name="paged_decode_bf16", kind="decode", dtype="bf16", batch=batch, hq=32,
                 hkv=8, d=128, block=64, top_k=32, ctx=tuple(ctx), steps=1,
                 seed=SEED_BASE + 2, sigma_q=1.0, a_q=1.0, delta=6.0, planted=(16, 16))
    return dataclasses.replace(w, **over)


def decode_1m_bf16(**over) -> Workload:
    """batch 1, 1048576 cached tokens, 64 query / 8 KV heads, d 128, block 128,
    top-k 16, 256 consecutive decode steps; 8 needle blocks per group in the first
    10% of the context with keys + 3 u."""
    w = Workload(name="decode_1m_bf16", kind="decode", dtype="bf16", batch=1, hq=64, hkv=8,
                 d=128, block=128, top_k=16, ctx=(1048576,), steps=256,
                 seed=SEED_BASE + 3, sigma_q=1.0, a_q=1.0, delta=3.0, planted=(8, 8),
                 planted_region=0.1)
    return dataclasses.replace(w, **over)


def varlen_decode_bf16(**over) -> Workload:
    """64 sequences with lengths log-uniform in [4096, 524288], 64 query / 4 KV heads,
    d 128, block 64, top-k 64; 0..32 planted blocks per (sequence, group), keys + 3 u."""
    batch = over.pop("batch", 64)
    lo, hi = over.pop("len_range", (4096, 524288))
    seed = over.get("seed", SEED_BASE + 4)
    if "ctx" in over:
        ctx = tuple(over.pop("ctx"))
    else:
        uu = uniform01((seed, 0x4C454E), batch)
        ctx = tuple(int(round(math.exp(math.log(lo) + float(x) * (math.log(hi) - math.log(lo)))))
                    for x in uu)
    w = Workload(name="varlen_decode_bf16", kind="decode", dtype="bf16", batch=batch, hq=64,
                 hkv=4, d=128, block=64, top_k=64, ctx=ctx, steps=1,
                 seed=SEED_BASE + 4, sigma_q=1.0, a_q=1.0, delta=3.0, planted=(0, 32))
    return dataclasses.replace(w, **over)


ALL = {
    "tiny_f32": tiny_f32,
    "prefill_bf16": prefill_bf16,
    "paged_decode_bf16": paged_decode_bf16,
    "decode_1m_bf16": decode_1m_bf16,
    "varlen_decode_bf16": varlen_decode_bf16,
}


# --------------------------------------------------------------------------
# small parameters (CPU)
# --------------------------------------------------------------------------
_T_Q, _T_K, _T_V, _T_U, _T_PLANT, _T_PERM, _T_QD, _T_TINY = range(1, 9)
_T_KI, _T_QI, _T_PTOK, _T_UI = range(9, 13)  # token-granular indexer inputs


@lru_cache(maxsize=64)
def _directions(w: Workload) -> torch.Tensor:
    """Unit planting direction u[b, g, :] (fp32, CPU)."""
    if w.tiny_q_hat:
        # mean over the group's heads of the last prefill query, normalised
        L = w.ctx[0]
        q_last = _raw_queries(w, 0, L - 1, L, "cpu").to(torch.float64)[0]  # [hq, d]
        out = torch.empty(w.batch, w.hkv, w.d, dtype=torch.float64)
        for g in range(w.hkv):
            m = q_last[g * w.group:(g + 1) * w.group].mean(0)
            out[0, g] = m / m.norm()
        return out.to(torch.float32)
    z = gauss((w.seed, _T_U), 0, w.batch * w.hkv * w.d, "cpu").to(torch.float64)
    z = z.view(w.batch, w.hkv, w.d)
    return (z / z.norm(dim=-1, keepdim=True)).to(torch.float32)


@lru_cache(maxsize=64)
def planted_blocks(w: Workload) -> List[List[List[int]]]:
    """planted[b][g] = sorted list of planted logical block ids (CPU)."""
    out = []
    for b in range(w.batch):
        n_blk = int(w.ctx[b] * w.planted_region) // w.block
        row = []
        for g in range(w.hkv):
            gen = cpu_generator(w.seed, _T_PLANT, b, g)
            lo, hi = w.planted
            cnt = lo if lo == hi else int(torch.randint(lo, hi + 1, (1,), generator=gen))
            cnt = min(cnt, n_blk)
            perm = torch.randperm(n_blk, generator=gen)[:cnt]
            row.append(sorted(int(x) for x in perm))
        out.append(row)
    return out


def _shift_rows(w: Workload, b: int, u0: int, u1: int) -> torch.Tensor:
    """[u1-u0, hkv, d] fp32 additive key shift (delta*u on planted blocks, else 0)."""
    u = _directions(w)[b]                               # [hkv, d]
    du = u * torch.tensor(w.delta, dtype=torch.float32)  # single fp32 rounding
    pos = torch.arange(u0, u1)
    mask = torch.zeros(u1 - u0, w.hkv, dtype=torch.float32)
    for g, blocks in enumerate(planted_blocks(w)[b]):
        for j in blocks:
            sel = (pos // w.block) == j
            mask[sel, g] = 1.0
    return mask[:, :, None] * du[None]


# --------------------------------------------------------------------------
# large tensors (any device, bit-identical)
# --------------------------------------------------------------------------
def keys(w: Workload, b: int, u0: int, u1: int, device="cpu") -> torch.Tensor:
    """Logical keys of sequence b at positions [u0, u1): [n, hkv, d] in w's dtype."""
    n = u1 - u0
    per = w.hkv * w.d
    z = gauss((w.seed, _T_K, b), u0 * per, n * per, device).view(n, w.hkv, w.d)
    if w.delta != 0.0:
        shift = _shift_rows(w, b, u0, u1)
        if bool(shift.any()):
            z = z + shift.to(device)
    return z.to(w.torch_dtype)


def values(w: Workload, b: int, u0: int, u1: int, device="cpu") -> torch.Tensor:
    """Logical values of sequence b at positions [u0, u1): [n, hkv, d]."""
    n = u1 - u0
    per = w.hkv * w.d
    z = gauss((w.seed, _T_V, b), u0 * per, n * per, device).view(n, w.hkv, w.d)
    return z.to(w.torch_dtype)


def _raw_queries(w: Workload, b: int, r0: int, r1: int, device) -> torch.Tensor:
    n = r1 - r0
    per = w.hq * w.d
    return gauss((w.seed, _T_Q, b), r0 * per, n * per, device).view(n, w.hq, w.d)


def _plant_queries(w: Workload, z: torch.Tensor, b: int) -> torch.Tensor:
    device = z.device
    if w.a_q != 0.0:
        u = _directions(w)[b]                                   # [hkv, d]
        au = (u * torch.tensor(w.a_q, dtype=torch.float32))     # [hkv, d]
        au = au.repeat_interleave(w.group, dim=0).to(device)    # [hq, d]
    if w.sigma_q != 1.0:
        z = z * torch.tensor(w.sigma_q, dtype=torch.float32, device=device)
    if w.a_q != 0.0:
        z = z + au[None]
    return z.to(w.torch_dtype)


def queries_prefill(w: Workload, b: int, r0: int, r1: int, device="cpu") -> torch.Tensor:
    """Prefill queries of sequence b at positions [r0, r1): [n, hq, d]."""
    return _plant_queries(w, _raw_queries(w, b, r0, r1, device), b)


def queries_decode(w: Workload, step: int, device="cpu", seqs=None) -> torch.Tensor:
    """Decode queries of step `step` for all (or the listed) sequences: [n, hq, d]."""
    seqs = range(w.batch) if seqs is None else seqs
    per = w.hq * w.d
    out = []
    for b in seqs:
        z = gauss((w.seed, _T_QD, b), step * per, per, device).view(1, w.hq, w.d)
        out.append(_plant_queries(w, z, b))
    return torch.cat(out, 0)


def new_tokens(w: Workload, step: int, device="cpu", seqs=None):
    """K and V rows appended by decode step `step`: two [n, hkv, d] tensors."""
    seqs = range(w.batch) if seqs is None else seqs
    ks, vs = [], []
    for b in seqs:
        p = w.ctx[b] + step
        ks.append(keys(w, b, p, p + 1, device))
        vs.append(values(w, b, p, p + 1, device))
    return torch.cat(ks, 0), torch.cat(vs, 0)


# --------------------------------------------------------------------------
# token-granular indexer inputs (synthetic: the indexer's weights are not given)
# --------------------------------------------------------------------------
@lru_cache(maxsize=64)
def planted_tokens(w: Workload, b: int, count: int = 32) -> List[int]:
    """Sorted positions of sequence b whose indexer keys lean toward the
    sequence's indexer direction (CPU)."""
    gen = cpu_generator(w.seed, _T_PTOK, b)
    n = w.total_len(b)
    return sorted(int(x) for x in torch.randperm(n, generator=gen)[:min(count, n)])


def _index_direction(w: Workload, b: int) -> torch.Tensor:
    z = gauss((w.seed, _T_UI, b), 0, w.d, "cpu").to(torch.float64)
    return (z / z.norm()).to(torch.float32)


def indexer_keys(w: Workload, b: int, u0: int, u1: int, device="cpu",
                 delta: float = 16.0) -> torch.Tensor:
    """Indexer keys of sequence b at positions [u0, u1): [n, d] in w's dtype,
    N(0, 1) plus delta along the sequence's indexer direction at the planted
    positions."""
    n = u1 - u0
    z = gauss((w.seed, _T_KI, b), u0 * w.d, n * w.d, device).view(n, w.d)
    pt = [p - u0 for p in planted_tokens(w, b) if u0 <= p < u1]
    if pt:
        z[torch.tensor(pt, device=z.device)] += (_index_direction(w, b) * delta).to(z.device)
    return z.to(w.torch_dtype)


def indexer_queries(w: Workload, step: int, heads: int, device="cpu",
                    a: float = 2.0) -> torch.Tensor:
    """Indexer queries of decode step `step`: [batch, heads, d], N(0, 1) plus a
    along the sequence's indexer direction in every head."""
    out = []
    for b in range(w.batch):
        z = gauss((w.seed, _T_QI, b), step * heads * w.d, heads * w.d, device).view(heads, w.d)
        out.append(z + (_index_direction(w, b) * a).to(z.device)[None])
    return torch.stack(out).to(w.torch_dtype)


# --------------------------------------------------------------------------
# paging
# --------------------------------------------------------------------------
@dataclasses.dataclass
class Paging:
    num_pages: int
    max_blocks: int
    table: torch.Tensor  # [batch, max_blocks] int32 (CPU), -1 where unused


def paging(w: Workload, spare_pages: int = 0) -> Paging:
    """Seeded random permutation of a global page pool, split per sequence."""
    need = [-(-w.total_len(b) // w.block) for b in range(w.batch)]
    total = sum(need) + spare_pages
    perm = torch.randperm(total, generator=cpu_generator(w.seed, _T_PERM))
    maxb = max(need)
    table = torch.full((w.batch, maxb), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n].to(torch.int32)
        off += n
    return Paging(num_pages=total, max_blocks=maxb, table=table)
