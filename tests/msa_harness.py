"""Test helpers: build paged caches through the library, run the oracle on the
same seeded inputs regenerated on the CPU, and compare by the parity rules.

Parity rules (bf16 / fp32 outputs, selected block indices):
  * indices bit-exact on every (row, group) whose oracle top-k gap is >= 1e-2;
    elsewhere every block the GPU picked must score within 1e-3 of the
    oracle's (k-1)-th best past-block score (several selections are correct
    when scores tie within fp32 rounding);
  * attention outputs compared element by element: bf16 max-abs 1e-2 and
    relative L2 5e-3; fp32 max-abs 1e-5;
  * centroids: fp32 relative 1e-6.
"""
from __future__ import annotations

import math
from typing import Dict, List, Sequence

import numpy as np
import torch

import block_sparse_gqa_mean_b200 as msa
import oracle
import workloads

GAP_MIN = 1e-2
TOL = {"bf16": dict(max_abs=1e-2, rel_l2=5e-3), "f32": dict(max_abs=1e-5, rel_l2=1e-5)}


def new_cache(w: workloads.Workload, paging: workloads.Paging, device="cuda") -> msa.PagedKVCache:
    cache = msa.PagedKVCache.allocate(
        batch=w.batch, num_pages=paging.num_pages, max_blocks_per_seq=paging.max_blocks,
        num_q_heads=w.hq, num_kv_heads=w.hkv, head_dim=w.d, block_size=w.block,
        dtype=w.torch_dtype, device=device)
    cache.page_table.copy_(paging.table.to(device))
    return cache


def append(cache: msa.PagedKVCache, w: workloads.Workload, before: Sequence[int],
           after: Sequence[int], device="cuda", k_rows=None, v_rows=None):
    """Append positions [before[b], after[b]) of every sequence through the library."""
    n = [a - b0 for b0, a in zip(before, after)]
    if k_rows is None:
        k_rows = torch.cat([workloads.keys(w, b, before[b], after[b], device) for b in range(w.batch)])
        v_rows = torch.cat([workloads.values(w, b, before[b], after[b], device) for b in range(w.batch)])
    cache.seq_lens.copy_(torch.tensor(list(after), dtype=torch.int32))
    cu = msa.cu_seqlens(n, device)
    msa.build_block_cache(cache, k_rows.contiguous(), v_rows.contiguous(), cu, max(n) if n else 0)


def fill_context(cache, w, device="cuda", per_call_tokens=1 << 22):
    """Append every sequence's cached context, a few sequences per call."""
    lens = [0] * w.batch
    for b in range(w.batch):
        L = w.ctx[b]
        step = max(1, per_call_tokens // (w.hkv * w.d))
        for u0 in range(0, L, step):
            u1 = min(L, u0 + step)
            before = list(lens)
            after = list(lens)
            after[b] = u1
            kr = workloads.keys(w, b, u0, u1, device)
            vr = workloads.values(w, b, u0, u1, device)
            # only sequence b grows in this call
            n = [after[i] - before[i] for i in range(w.batch)]
            cache.seq_lens.copy_(torch.tensor(after, dtype=torch.int32))
            msa.build_block_cache(cache, kr, vr, msa.cu_seqlens(n, device), max(n))
            lens = after
    return lens


def read_pages(cache: msa.PagedKVCache, b: int, L: int, which="k") -> torch.Tensor:
    """Logical [L, Hkv, d] rows of sequence b gathered back from the pages (CPU)."""
    pages = (cache.k_pages if which == "k" else cache.v_pages)
    nblk = -(-L // cache.block_size)
    ids = cache.page_table[b, :nblk].long()
    blocks = pages[ids]                                # [nblk, Hkv, B, d]
    return blocks.permute(0, 2, 1, 3).reshape(nblk * cache.block_size, cache.num_kv_heads,
                                              cache.head_dim)[:L].cpu()


def oracle_rows(w: workloads.Workload, b: int, L: int, rows_pos: np.ndarray, Q,
                idx=None) -> Dict[str, np.ndarray]:
    """Oracle for query rows of sequence b (cache of L tokens) at positions rows_pos."""
    K = workloads.keys(w, b, 0, L)
    V = workloads.values(w, b, 0, L)
    if idx is None:
        return oracle.forward(Q, K, V, rows_pos, w.block, w.top_k, w.softmax_scale)
    O, lse = oracle.attend(Q, K, V, rows_pos, idx, w.block, w.softmax_scale)
    return {"out": O, "lse": lse}


def check_index_invariants(idx: np.ndarray, pos: np.ndarray, block: int, k: int):
    """Ascending, unique, own block present, no future block, size min(k, b+1)."""
    for r in range(idx.shape[0]):
        own = pos[r] // block
        for g in range(idx.shape[1]):
            row = idx[r, g]
            valid = row[row >= 0]
            assert len(valid) == min(k, own + 1), (r, g, row)
            assert np.all(row[len(valid):] == -1)
            assert np.all(np.diff(valid) > 0)
            assert valid[-1] == own and valid[0] >= 0


def check_selection(gpu_idx: np.ndarray, orc: Dict[str, np.ndarray], pos: np.ndarray, k: int,
                    block: int) -> Dict[str, float]:
    """Bit-exact where the oracle gap is >= GAP_MIN, near-optimal elsewhere."""
    check_index_invariants(gpu_idx, pos, block, k)
    gap, oidx, S = orc["gap"], orc["idx"], orc["scores"]
    protected = gap >= GAP_MIN
    mism = (gpu_idx != oidx).any(-1)
    assert not np.any(mism & protected), np.argwhere(mism & protected)[:5]
    for r, g in np.argwhere(mism):
        own = pos[r] // block
        past = np.sort(S[r, g, :own])[::-1]
        thresh = past[k - 2]
        chosen = [j for j in gpu_idx[r, g] if 0 <= j < own]
        assert all(S[r, g, j] >= thresh - 1e-3 for j in chosen), (r, g)
    return {"rows": float(gap.size), "protected_frac": float(protected.mean()),
            "mismatch_frac": float(mism.mean())}


def compare(out_gpu: torch.Tensor, ref: np.ndarray, dtype: str):
    o = out_gpu.detach().float().cpu().double().numpy()
    err = np.abs(o - ref)
    max_abs = float(err.max())
    rel = float(np.linalg.norm(o - ref) / max(np.linalg.norm(ref), 1e-30))
    tol = TOL[dtype]
    if not (max_abs <= tol["max_abs"] and rel <= tol["rel_l2"]):
        i = np.unravel_index(int(err.argmax()), err.shape)
        raise AssertionError(f"max_abs {max_abs:.4g} rel_l2 {rel:.4g} worst at {i}: "
                             f"gpu {o[i]!r} oracle {ref[i]!r}")
    return max_abs, rel
