"""CPU fp64 oracle for block-sparse GQA attention with a mean-pooled block cache.

TEST INFRASTRUCTURE ONLY: the test suite, the package's smoke check and the
benchmark's CPU-baseline leg are the only callers. The product path (the CUDA
library and its Python binding) never imports this package.

The arithmetic lives in ``msa_oracle.cpp`` (plain C++17 + OpenMP, fp64). This
module converts arrays and calls it. Every function takes the *logical*
(unpaged) tensors of one sequence:

  K, V : [L, Hkv, d]     keys / values at positions 0 .. L-1
  Q    : [R, Hq, d]      query rows, row r at position pos[r]

as fp32 arrays or bf16 bit patterns (torch.bfloat16 tensors or uint16 numpy
arrays); elements are widened to double on use.

Citations (page title, section):
  * centroids  - "Art of Focus: Ling 2.0 ...", "Summarizing the Breakthrough":
                 blocks are aggregated into representations kept in the cache
                 (read here as the mean of the keys present).
  * scores, select - "MiniMax Sparse Attention", method paragraph: the index
                 branch scores KV blocks and takes a top-k subset per GQA group;
                 results paragraph: the top-k is exp-free.
  * attend     - "MiniMax Sparse Attention", method paragraph (exact blockwise
                 sparse attention over the chosen blocks) and "Sparse Attention
                 + Linear Backbones", section 5.5 (softmax(q k^T / sqrt(d)) v).
  * gate       - "Sparse Attention for Long-Context LLMs: Evolution and
                 Practical Deployment", section 4.3, step 6 of the computation
                 flow: O = Gate * A + (1 - Gate) * X, the gate a scalar or
                 varying with the dimension (X given by the caller).
  * token_scores, token_select, attend_tokens - the token-granular variant of
                 "Sparse Attention + Linear Backbones: How LLM Long-Context
                 Architectures Are Evolving", sections 5.1-5.3 and 5.5: a
                 lightweight multi-head indexer without positional encoding
                 rates all earlier positions, the top-K positions are
                 kept, and the main attention runs over those positions only.
                 The page leaves the indexer's form open; the reading here
                 mirrors the block path: s(t, u) = sum over indexer heads h of
                 qI[t, h] . kI[u] for u <= t, exp-free, the query's own
                 position always kept, ties to the lower position (pure numpy,
                 fp64).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (g++, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.orc_centroids.restype = _I64
        lib.orc_centroids.argtypes = [_P, _I32, _I64, _I32, _I32, _I32, _P]
        lib.orc_scores.restype = None
        lib.orc_scores.argtypes = [_P, _I32, _I64, _P, _I32, _I32, _I32, _I32, _P, _I64, _P]
        lib.orc_select.restype = None
        lib.orc_select.argtypes = [_P, _I64, _P, _I32, _I64, _I32, _I32, _P, _P]
        lib.orc_attend.restype = None
        lib.orc_attend.argtypes = [_P, _P, _P, _I32, _I64, _P, _I64, _I32, _I32, _I32, _I32, _P,
                                   _I32, ctypes.c_double, _P, _P]
        lib.orc_num_threads.restype = _I32
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().orc_num_threads())


def _elems(x):
    """(contiguous numpy array, dtype code) for fp32 or bf16-bit input."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return np.ascontiguousarray(x.view(torch.int16).numpy().view(np.uint16)), 1
            return np.ascontiguousarray(x.to(torch.float32).numpy()), 0
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), 1
    return np.ascontiguousarray(x, dtype=np.float32), 0


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def centroids(K, block: int) -> np.ndarray:
    """[ceil(L/B), Hkv, d] fp64 mean of the keys present in each block."""
    k, dt = _elems(K)
    L, hkv, d = k.shape
    nblk = -(-L // block)
    C = np.empty((nblk, hkv, d), dtype=np.float64)
    _load().orc_centroids(_ptr(k), dt, L, hkv, d, block, _ptr(C))
    return C


def scores(Q, pos, C: np.ndarray, block: int) -> np.ndarray:
    """[R, Hkv, nblk] fp64 block scores; NaN outside the candidate set."""
    q, dt = _elems(Q)
    R, hq, d = q.shape
    nblk, hkv, _ = C.shape
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    C = np.ascontiguousarray(C, dtype=np.float64)
    S = np.empty((R, hkv, nblk), dtype=np.float64)
    _load().orc_scores(_ptr(q), dt, R, _ptr(pos), hq, hkv, d, block, _ptr(C), nblk, _ptr(S))
    return S


def select(S: np.ndarray, pos, block: int, top_k: int):
    """(idx [R, Hkv, k] int32 ascending, -1 padded; gap [R, Hkv] fp64)."""
    S = np.ascontiguousarray(S, dtype=np.float64)
    R, hkv, nblk = S.shape
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    idx = np.empty((R, hkv, top_k), dtype=np.int32)
    gap = np.empty((R, hkv), dtype=np.float64)
    _load().orc_select(_ptr(S), R, _ptr(pos), hkv, nblk, block, top_k, _ptr(idx), _ptr(gap))
    return idx, gap


def attend(Q, K, V, pos, idx, block: int, scale: float):
    """(O [R, Hq, d] fp64, lse [R, Hq] fp64) of exact attention over idx's blocks."""
    q, dq = _elems(Q)
    k, dk = _elems(K)
    v, dv = _elems(V)
    if not (dq == dk == dv):
        raise TypeError("Q, K, V must share one element type")
    R, hq, d = q.shape
    L, hkv, _ = k.shape
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    top_k = idx.shape[-1]
    O = np.empty((R, hq, d), dtype=np.float64)
    lse = np.empty((R, hq), dtype=np.float64)
    _load().orc_attend(_ptr(q), _ptr(k), _ptr(v), dq, R, _ptr(pos), L, hq, hkv, d, block,
                       _ptr(idx), top_k, float(scale), _ptr(O), _ptr(lse))
    return O, lse


def forward(Q, K, V, pos, block: int, top_k: int, scale: float) -> Dict[str, np.ndarray]:
    """Whole path for one sequence: centroids -> scores -> top-k -> attention."""
    C = centroids(K, block)
    S = scores(Q, pos, C, block)
    idx, gap = select(S, pos, block, top_k)
    O, lse = attend(Q, K, V, pos, idx, block, scale)
    return {"centroids": C, "scores": S, "idx": idx, "gap": gap, "out": O, "lse": lse}


def gate(A, g, X) -> np.ndarray:
    """O = g * A + (1 - g) * X in fp64, literally. A, X: [R, Hq, d]; g: [R, Hq]
    (one value per row and head) or [R, Hq, d]."""
    A = np.asarray(A, dtype=np.float64)
    X = np.asarray(_widen(X), dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    if g.ndim == A.ndim - 1:
        g = g[..., None]
    return g * A + (1.0 - g) * X


def _widen(x):
    """bf16 torch tensors / uint16 bit patterns -> float64 values."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").double().numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


# --------------------------------------------------------------------------
# token-granular variant (indexer over every position, top-K tokens)
# --------------------------------------------------------------------------
def token_scores(QI, KI, pos) -> np.ndarray:
    """s[r, u] = sum_h QI[r, h] . KI[u] in fp64 for u <= pos[r]; -inf after.
    QI: [R, Hi, di] indexer queries; KI: [L, di] indexer keys (one per position)."""
    qi = np.asarray(_widen(QI), dtype=np.float64)
    ki = np.asarray(_widen(KI), dtype=np.float64)
    pos = np.asarray(pos, dtype=np.int64)
    S = np.einsum("rhd,ud->ru", qi, ki)
    future = np.arange(ki.shape[0])[None, :] > pos[:, None]
    S[future] = -np.inf
    return S


def token_select(S: np.ndarray, pos, top_k: int):
    """(idx [R, top_k] int32 ascending, -1 padded; gap [R]) of the kept positions:
    the own position pos[r] plus the top_k - 1 best earlier positions (scores
    descending, ties to the lower position). gap = score of the last kept
    earlier position minus the best dropped one (+inf when nothing is dropped)."""
    pos = np.asarray(pos, dtype=np.int64)
    R = S.shape[0]
    idx = np.full((R, top_k), -1, dtype=np.int32)
    gap = np.full(R, np.inf)
    for r in range(R):
        t = int(pos[r])
        cand = np.arange(t)                                # earlier positions
        order = cand[np.lexsort((cand, -S[r, :t]))] if t else cand
        take = min(top_k - 1, t)
        kept = np.sort(np.concatenate([order[:take], [t]]))
        idx[r, :len(kept)] = kept
        if 0 < take < t:
            gap[r] = S[r, order[take - 1]] - S[r, order[take]]
    return idx, gap


def attend_tokens(Q, K, V, pos, tok_idx, scale: float):
    """(O [R, Hq, d], lse [R, Hq]) of exact attention of row r over the listed
    positions u (tok_idx[r], -1 padding, a repeat counts once, u <= pos[r]),
    the query head h reading KV head h // (Hq // Hkv)."""
    q = np.asarray(_widen(Q), dtype=np.float64)
    k = np.asarray(_widen(K), dtype=np.float64)
    v = np.asarray(_widen(V), dtype=np.float64)
    pos = np.asarray(pos, dtype=np.int64)
    R, hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    O = np.zeros((R, hq, d))
    lse = np.full((R, hq), -np.inf)
    for r in range(R):
        u = np.unique(tok_idx[r][(tok_idx[r] >= 0) & (tok_idx[r] <= pos[r])])
        if len(u) == 0:
            continue
        for h in range(hq):
            logit = scale * (k[u, h // G] @ q[r, h])
            m = logit.max()
            w = np.exp(logit - m)
            O[r, h] = (w / w.sum()) @ v[u, h // G]
            lse[r, h] = m + np.log(w.sum())
    return O, lse
