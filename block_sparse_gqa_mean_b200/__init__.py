"""Block-sparse GQA attention with a mean-pooled block cache, for B200 (sm_100a).

Thin Python binding of libmsa.so (include/msa.h). It only marshals torch CUDA
tensors into the C ABI: device pointers, host integers and the current CUDA
stream. Every step of the computation runs in the library's CUDA kernels;
there is no CPU or framework fallback, and importing the binding without the
built library raises.

    cache = PagedKVCache.allocate(batch=1, num_pages=..., max_blocks_per_seq=...,
                                  num_q_heads=32, num_kv_heads=4, head_dim=128,
                                  block_size=128, dtype=torch.bfloat16)
    cache.page_table.copy_(table); cache.seq_lens.copy_(lens_after_append)
    build_block_cache(cache, k_new, v_new, cu_new, max_new_per_seq)
    idx, _ = select_topk(cache, q, top_k=16, cu_q=cu_q, max_rows_per_seq=T)
    out, lse = sparse_attn_prefill(cache, q, idx, cu_q=cu_q, max_rows_per_seq=T)
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MSA_LIBRARY may name another build of the library, e.g. the bounds-checked
# libmsa_debug.so (python -m block_sparse_gqa_mean_b200.build --debug-bounds).
LIB_PATH = os.environ.get("MSA_LIBRARY") or os.path.join(_PKG, "libmsa.so")
DEBUG_LIB_PATH = os.path.join(_PKG, "libmsa_debug.so")

MSA_OK, MSA_ERR_INVALID_ARG, MSA_ERR_UNSUPPORTED, MSA_ERR_WORKSPACE, MSA_ERR_CUDA = range(5)
MSA_DTYPE_BF16, MSA_DTYPE_F32 = 0, 1
MSA_OP_SELECT, MSA_OP_PREFILL, MSA_OP_DECODE, MSA_OP_SELECT_TOKENS = 0, 1, 2, 3
MSA_DEV_BAD_PAGE, MSA_DEV_BAD_LENGTH, MSA_DEV_BAD_INDEX, MSA_DEV_TIMEOUT = 1, 2, 4, 8
MSA_DEV_BOUNDS = 0x10
MSA_BUILD_DEBUG_BOUNDS = 1

EXPORTS = ("msa_build_block_cache", "msa_select_topk", "msa_sparse_attn_prefill",
           "msa_sparse_attn_decode", "msa_sparse_attn_prefill_gated",
           "msa_sparse_attn_decode_gated", "msa_sparse_attn_decode_noalloc", "msa_workspace_size",
           "msa_status_string", "msa_version", "msa_select_tokens", "msa_sparse_attn_decode_tokens",
           "msa_select_topk_range", "msa_select_merge", "msa_sparse_attn_decode_range",
           "msa_lse_merge", "msa_select_tokens_rows", "msa_sparse_attn_prefill_tokens",
           "msa_build_flags", "msa_selftest_bounded_wait")


class MsaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class _PagedKV(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32),
        ("k_pages", ctypes.c_void_p),
        ("v_pages", ctypes.c_void_p),
        ("centroids", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
        ("status_word", ctypes.c_void_p),
    ]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmsa.so. Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libmsa.so not found at {path}; build it with "
                          "`python -m block_sparse_gqa_mean_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    KV = ctypes.POINTER(_PagedKV)
    lib.msa_build_block_cache.argtypes = [KV, P, P, P, I32, P]
    lib.msa_select_topk.argtypes = [KV, P, P, I32, I32, I32, P, P, P, SZ, P]
    lib.msa_sparse_attn_prefill.argtypes = [KV, P, P, I32, I32, P, I32, ctypes.c_float, P, P, P,
                                            SZ, P]
    lib.msa_sparse_attn_decode.argtypes = [KV, P, P, I32, ctypes.c_float, P, P, P, SZ, P]
    lib.msa_sparse_attn_decode_noalloc.argtypes = [KV, P, P, I32, ctypes.c_float, P, P, P]
    lib.msa_sparse_attn_prefill_gated.argtypes = [KV, P, P, I32, I32, P, I32, ctypes.c_float, P,
                                                  I32, P, P, P, P, SZ, P]
    lib.msa_sparse_attn_decode_gated.argtypes = [KV, P, P, I32, ctypes.c_float, P, I32, P, P, P, P,
                                                 SZ, P]
    lib.msa_select_tokens.argtypes = [KV, P, P, I32, I32, P, P, SZ, P]
    lib.msa_sparse_attn_decode_tokens.argtypes = [KV, P, P, I32, ctypes.c_float, P, P, P]
    lib.msa_select_topk_range.argtypes = [KV, P, I32, I32, I32, P, P, SZ, P]
    lib.msa_select_merge.argtypes = [KV, P, I32, I32, P, P, P]
    lib.msa_sparse_attn_decode_range.argtypes = [KV, P, P, I32, I32, I32, ctypes.c_float, P, P, P,
                                                 SZ, P]
    lib.msa_lse_merge.argtypes = [P, P, I32, I32, I32, I32, P, P, P]
    lib.msa_select_tokens_rows.argtypes = [KV, P, P, P, I32, I32, I32, P, P, SZ, P]
    lib.msa_sparse_attn_prefill_tokens.argtypes = [KV, P, P, I32, P, I32, ctypes.c_float, P, P, P]
    lib.msa_workspace_size.argtypes = [ctypes.c_int, KV, I32, I32, I32]
    lib.msa_workspace_size.restype = SZ
    lib.msa_status_string.argtypes = [ctypes.c_int]
    lib.msa_status_string.restype = ctypes.c_char_p
    lib.msa_version.restype = I32
    lib.msa_build_flags.restype = I32
    lib.msa_selftest_bounded_wait.argtypes = [I32, P, P]
    lib.msa_selftest_bounded_wait.restype = ctypes.c_int
    for name in ("msa_build_block_cache", "msa_select_topk", "msa_sparse_attn_prefill",
                 "msa_sparse_attn_decode", "msa_sparse_attn_prefill_gated",
                 "msa_sparse_attn_decode_gated", "msa_sparse_attn_decode_noalloc",
                 "msa_select_tokens", "msa_sparse_attn_decode_tokens", "msa_select_topk_range",
                 "msa_select_merge", "msa_sparse_attn_decode_range", "msa_lse_merge",
                 "msa_select_tokens_rows", "msa_sparse_attn_prefill_tokens"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().msa_status_string(status).decode()


def selftest_bounded_wait(which: int, status_word: torch.Tensor, stream=None) -> None:
    """Run one of the library's bounded device waits on something that is
    never completed (0: an mbarrier phase, 1: a flag another CTA would
    publish); after about a second it sets MSA_DEV_TIMEOUT in status_word
    (a one-element int32 CUDA tensor) and returns."""
    _require_cuda(status_word)
    _check(load_library().msa_selftest_bounded_wait(int(which), _ptr(status_word), _stream(stream)),
           "msa_selftest_bounded_wait")


def build_flags() -> int:
    """MSA_BUILD_* bits of the loaded library (MSA_BUILD_DEBUG_BOUNDS for
    the bounds-checked build)."""
    return int(load_library().msa_build_flags())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != MSA_OK:
        raise MsaError(status, what)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


@dataclasses.dataclass
class PagedKVCache:
    """Caller-owned paged cache: K/V pages, fp32 centroids (block cache sharing the
    page ids), page table, sequence lengths and the device status word."""
    k_pages: torch.Tensor      # [num_pages, Hkv, B, d]
    v_pages: torch.Tensor      # [num_pages, Hkv, B, d]
    centroids: torch.Tensor    # [num_pages, Hkv, d] fp32
    page_table: torch.Tensor   # [batch, max_blocks_per_seq] int32
    seq_lens: torch.Tensor     # [batch] int32
    status_word: torch.Tensor  # [4] int32 (first word used)
    num_q_heads: int

    @classmethod
    def allocate(cls, batch: int, num_pages: int, max_blocks_per_seq: int, num_q_heads: int,
                 num_kv_heads: int, head_dim: int, block_size: int,
                 dtype: torch.dtype = torch.bfloat16, device="cuda") -> "PagedKVCache":
        kp = torch.zeros(num_pages, num_kv_heads, block_size, head_dim, dtype=dtype, device=device)
        vp = torch.zeros_like(kp)
        cen = torch.zeros(num_pages, num_kv_heads, head_dim, dtype=torch.float32, device=device)
        pt = torch.full((batch, max_blocks_per_seq), -1, dtype=torch.int32, device=device)
        sl = torch.zeros(batch, dtype=torch.int32, device=device)
        st = torch.zeros(4, dtype=torch.int32, device=device)
        return cls(kp, vp, cen, pt, sl, st, num_q_heads)

    @property
    def num_kv_heads(self) -> int:
        return self.k_pages.shape[1]

    @property
    def block_size(self) -> int:
        return self.k_pages.shape[2]

    @property
    def head_dim(self) -> int:
        return self.k_pages.shape[3]

    @property
    def batch(self) -> int:
        return self.page_table.shape[0]

    @property
    def dtype(self) -> torch.dtype:
        return self.k_pages.dtype

    def struct(self) -> _PagedKV:
        _require_cuda(self.k_pages, self.v_pages, self.centroids, self.page_table, self.seq_lens,
                      self.status_word)
        if self.k_pages.dtype == torch.bfloat16:
            dt = MSA_DTYPE_BF16
        elif self.k_pages.dtype == torch.float32:
            dt = MSA_DTYPE_F32
        else:
            raise TypeError("K/V pages must be bf16 or fp32")
        return _PagedKV(dt, self.num_q_heads, self.num_kv_heads, self.head_dim, self.block_size,
                        self.batch, self.k_pages.shape[0], self.page_table.shape[1],
                        self.k_pages.data_ptr(), self.v_pages.data_ptr(),
                        self.centroids.data_ptr(), self.page_table.data_ptr(),
                        self.seq_lens.data_ptr(), self.status_word.data_ptr())

    def device_status(self) -> int:
        """Read (synchronously) the device status word."""
        return int(self.status_word[0].item()) & 0xFFFFFFFF

    def clear_status(self):
        self.status_word.zero_()


def workspace_size(op: int, cache: PagedKVCache, num_rows: int, max_rows_per_seq: int,
                   top_k: int) -> int:
    kv = cache.struct()
    return int(load_library().msa_workspace_size(op, ctypes.byref(kv), num_rows, max_rows_per_seq,
                                                 top_k))


def _workspace(op, cache, num_rows, max_rows, top_k, workspace):
    need = workspace_size(op, cache, num_rows, max_rows, top_k)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=cache.k_pages.device)
    return workspace, workspace.numel() * workspace.element_size()


def build_block_cache(cache: PagedKVCache, k_new: torch.Tensor, v_new: torch.Tensor,
                      cu_new: torch.Tensor, max_new_per_seq: int, stream=None) -> None:
    """Append k_new/v_new rows (cache.seq_lens already counts them) and re-pool
    the centroids of every touched block."""
    lib = load_library()
    _require_cuda(k_new, v_new, cu_new)
    kv = cache.struct()
    _check(lib.msa_build_block_cache(ctypes.byref(kv), _ptr(k_new), _ptr(v_new), _ptr(cu_new),
                                     int(max_new_per_seq), _stream(stream)),
           "msa_build_block_cache")


def select_topk(cache: PagedKVCache, q: torch.Tensor, top_k: int,
                cu_q: Optional[torch.Tensor] = None, max_rows_per_seq: int = 1,
                block_idx: Optional[torch.Tensor] = None, block_score: Optional[torch.Tensor] = None,
                want_scores: bool = False, workspace: Optional[torch.Tensor] = None,
                stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Per-group top-k block selection. cu_q None = decode (one row per sequence)."""
    lib = load_library()
    _require_cuda(q, cu_q, block_idx, block_score)
    rows = q.shape[0]
    if block_idx is None:
        block_idx = torch.empty(rows, cache.num_kv_heads, top_k, dtype=torch.int32, device=q.device)
    if block_score is None and want_scores:
        block_score = torch.empty(rows, cache.num_kv_heads, top_k, dtype=torch.float32,
                                  device=q.device)
    mr = 1 if cu_q is None else max_rows_per_seq
    ws, ws_bytes = _workspace(MSA_OP_SELECT, cache, rows, mr, top_k, workspace)
    kv = cache.struct()
    _check(lib.msa_select_topk(ctypes.byref(kv), _ptr(q), _ptr(cu_q), rows, mr, top_k,
                               _ptr(block_idx), _ptr(block_score), _ptr(ws), ws_bytes,
                               _stream(stream)), "msa_select_topk")
    return block_idx, block_score


def sparse_attn_prefill(cache: PagedKVCache, q: torch.Tensor, block_idx: torch.Tensor,
                        cu_q: torch.Tensor, max_rows_per_seq: int,
                        softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                        lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                        workspace: Optional[torch.Tensor] = None, stream=None,
                        gate: Optional[torch.Tensor] = None, x: Optional[torch.Tensor] = None):
    """Exact attention of the query rows over their selected blocks. With `gate`
    (fp32, [rows, Hq] or [rows, Hq, d]) and `x` ([rows, Hq, d]) the output is
    gate * attention + (1 - gate) * x, fused into the kernel's epilogue."""
    lib = load_library()
    _require_cuda(q, block_idx, cu_q, out, lse, gate, x)
    rows, top_k = q.shape[0], block_idx.shape[-1]
    scale = 1.0 / math.sqrt(cache.head_dim) if softmax_scale is None else softmax_scale
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(rows, q.shape[1], dtype=torch.float32, device=q.device)
    ws, ws_bytes = _workspace(MSA_OP_PREFILL, cache, rows, max_rows_per_seq, top_k, workspace)
    kv = cache.struct()
    if gate is not None:
        per_dim = _gate_layout(gate, x, q)
        _check(lib.msa_sparse_attn_prefill_gated(ctypes.byref(kv), _ptr(q), _ptr(cu_q), rows,
                                                 max_rows_per_seq, _ptr(block_idx), top_k, scale,
                                                 _ptr(gate), per_dim, _ptr(x), _ptr(out),
                                                 _ptr(lse), _ptr(ws), ws_bytes, _stream(stream)),
               "msa_sparse_attn_prefill_gated")
        return out, lse
    _check(lib.msa_sparse_attn_prefill(ctypes.byref(kv), _ptr(q), _ptr(cu_q), rows,
                                       max_rows_per_seq, _ptr(block_idx), top_k, scale, _ptr(out),
                                       _ptr(lse), _ptr(ws), ws_bytes, _stream(stream)),
           "msa_sparse_attn_prefill")
    return out, lse


def sparse_attn_decode(cache: PagedKVCache, q: torch.Tensor, block_idx: torch.Tensor,
                       softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                       workspace: Optional[torch.Tensor] = None, stream=None,
                       gate: Optional[torch.Tensor] = None, x: Optional[torch.Tensor] = None):
    """Attention of one new query per sequence (at seq_lens-1) over its selected
    blocks; `gate` and `x` as for sparse_attn_prefill."""
    lib = load_library()
    _require_cuda(q, block_idx, out, lse, gate, x)
    top_k = block_idx.shape[-1]
    scale = 1.0 / math.sqrt(cache.head_dim) if softmax_scale is None else softmax_scale
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device)
    ws, ws_bytes = _workspace(MSA_OP_DECODE, cache, q.shape[0], 1, top_k, workspace)
    kv = cache.struct()
    if gate is not None:
        per_dim = _gate_layout(gate, x, q)
        _check(lib.msa_sparse_attn_decode_gated(ctypes.byref(kv), _ptr(q), _ptr(block_idx), top_k,
                                                scale, _ptr(gate), per_dim, _ptr(x), _ptr(out),
                                                _ptr(lse), _ptr(ws), ws_bytes, _stream(stream)),
               "msa_sparse_attn_decode_gated")
        return out, lse
    _check(lib.msa_sparse_attn_decode(ctypes.byref(kv), _ptr(q), _ptr(block_idx), top_k, scale,
                                      _ptr(out), _ptr(lse), _ptr(ws), ws_bytes, _stream(stream)),
           "msa_sparse_attn_decode")
    return out, lse


def _gate_layout(gate: torch.Tensor, x: Optional[torch.Tensor], q: torch.Tensor) -> int:
    """Checks the gate and x tensors; returns 1 for a per-coordinate gate."""
    if x is None or x.shape != q.shape or x.dtype != q.dtype or not x.is_contiguous():
        raise ValueError("x must be a contiguous tensor shaped and typed like q")
    if gate.dtype != torch.float32 or not gate.is_contiguous():
        raise ValueError("gate must be a contiguous fp32 tensor")
    if tuple(gate.shape) == tuple(q.shape):
        return 1
    if tuple(gate.shape) == tuple(q.shape[:2]):
        return 0
    raise ValueError("gate must be shaped [rows, Hq] or [rows, Hq, d]")


def sparse_attn_decode_noalloc(cache: PagedKVCache, q: torch.Tensor, block_idx: torch.Tensor,
                               out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                               softmax_scale: Optional[float] = None, stream=None):
    """sparse_attn_decode for callers that cannot allocate device memory: the
    caller passes the outputs, and the attention's scratch (one part and flag
    per resident CTA, at most ~5 MiB) is the library's own 8 MiB device array
    (shared by every call on the device, so calls must not overlap on the
    GPU)."""
    lib = load_library()
    _require_cuda(q, block_idx, out, lse)
    top_k = block_idx.shape[-1]
    scale = 1.0 / math.sqrt(cache.head_dim) if softmax_scale is None else softmax_scale
    kv = cache.struct()
    _check(lib.msa_sparse_attn_decode_noalloc(ctypes.byref(kv), _ptr(q), _ptr(block_idx), top_k,
                                              scale, _ptr(out), _ptr(lse), _stream(stream)),
           "msa_sparse_attn_decode_noalloc")
    return out, lse


def select_tokens(cache: PagedKVCache, ki_pages: torch.Tensor, qi: torch.Tensor, top_k: int,
                  tok_idx: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Token-granular selection for one new query per sequence (at seq_lens-1):
    ki_pages [num_pages, block_size, head_dim] (one indexer key per position,
    paged with the cache's page table), qi [batch, num_index_heads, head_dim].
    Returns tok_idx [batch, top_k] int32: the kept positions ascending (the
    query's own position last), -1 padded."""
    lib = load_library()
    _require_cuda(ki_pages, qi, tok_idx)
    if tok_idx is None:
        tok_idx = torch.empty(qi.shape[0], top_k, dtype=torch.int32, device=qi.device)
    ws, ws_bytes = _workspace(MSA_OP_SELECT_TOKENS, cache, qi.shape[0], 1, top_k, workspace)
    kv = cache.struct()
    _check(lib.msa_select_tokens(ctypes.byref(kv), _ptr(ki_pages), _ptr(qi), qi.shape[1], top_k,
                                 _ptr(tok_idx), _ptr(ws), ws_bytes, _stream(stream)),
           "msa_select_tokens")
    return tok_idx


def select_tokens_rows(cache: PagedKVCache, ki_pages: torch.Tensor, qi: torch.Tensor, top_k: int,
                       cu_q: torch.Tensor, max_rows_per_seq: int,
                       tok_idx: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Token-granular selection for many rows per sequence (prefill): qi
    [rows, num_index_heads, head_dim]; the rows of sequence b are its last n_b
    positions (cu_q as for select_topk). Returns tok_idx [rows, top_k]."""
    lib = load_library()
    _require_cuda(ki_pages, qi, cu_q, tok_idx)
    rows = qi.shape[0]
    if tok_idx is None:
        tok_idx = torch.empty(rows, top_k, dtype=torch.int32, device=qi.device)
    ws, ws_bytes = _workspace(MSA_OP_SELECT_TOKENS, cache, rows, max(2, max_rows_per_seq), top_k,
                              workspace)
    kv = cache.struct()
    _check(lib.msa_select_tokens_rows(ctypes.byref(kv), _ptr(ki_pages), _ptr(qi), _ptr(cu_q), rows,
                                      qi.shape[1], top_k, _ptr(tok_idx), _ptr(ws), ws_bytes,
                                      _stream(stream)), "msa_select_tokens_rows")
    return tok_idx


def sparse_attn_prefill_tokens(cache: PagedKVCache, q: torch.Tensor, tok_idx: torch.Tensor,
                               cu_q: torch.Tensor, softmax_scale: Optional[float] = None,
                               out: Optional[torch.Tensor] = None,
                               lse: Optional[torch.Tensor] = None, stream=None):
    """Attention of each prefill row over its own kept positions."""
    lib = load_library()
    _require_cuda(q, tok_idx, cu_q, out, lse)
    top_k = tok_idx.shape[-1]
    scale = 1.0 / math.sqrt(cache.head_dim) if softmax_scale is None else softmax_scale
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device)
    kv = cache.struct()
    _check(lib.msa_sparse_attn_prefill_tokens(ctypes.byref(kv), _ptr(q), _ptr(cu_q), q.shape[0],
                                              _ptr(tok_idx), top_k, scale, _ptr(out), _ptr(lse),
                                              _stream(stream)), "msa_sparse_attn_prefill_tokens")
    return out, lse


def sparse_attn_decode_tokens(cache: PagedKVCache, q: torch.Tensor, tok_idx: torch.Tensor,
                              softmax_scale: Optional[float] = None,
                              out: Optional[torch.Tensor] = None,
                              lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                              stream=None):
    """Attention of one new query per sequence over the positions in tok_idx."""
    lib = load_library()
    _require_cuda(q, tok_idx, out, lse)
    top_k = tok_idx.shape[-1]
    scale = 1.0 / math.sqrt(cache.head_dim) if softmax_scale is None else softmax_scale
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device)
    kv = cache.struct()
    _check(lib.msa_sparse_attn_decode_tokens(ctypes.byref(kv), _ptr(q), _ptr(tok_idx), top_k,
                                             scale, _ptr(out), _ptr(lse), _stream(stream)),
           "msa_sparse_attn_decode_tokens")
    return out, lse


# ---------------------------------------------------------------------------
# context-sharded decode (blocks of every sequence split over ranks by range)
# ---------------------------------------------------------------------------
def select_topk_range(cache: PagedKVCache, q: torch.Tensor, top_k: int, block_lo: int,
                      block_hi: int, cand_keys: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """This rank's best top_k-1 candidates among blocks [block_lo, block_hi) of
    every sequence's decode row: [batch, Hkv, top_k-1] selection keys (int64
    bit patterns of the library's unsigned keys, descending, 0 padded)."""
    lib = load_library()
    _require_cuda(q, cand_keys)
    if cand_keys is None:
        cand_keys = torch.zeros(q.shape[0], cache.num_kv_heads, max(top_k - 1, 1),
                                dtype=torch.int64, device=q.device)
    ws, ws_bytes = _workspace(MSA_OP_SELECT, cache, q.shape[0], 1, top_k, workspace)
    kv = cache.struct()
    _check(lib.msa_select_topk_range(ctypes.byref(kv), _ptr(q), int(block_lo), int(block_hi),
                                     top_k, _ptr(cand_keys), _ptr(ws), ws_bytes, _stream(stream)),
           "msa_select_topk_range")
    return cand_keys


def select_merge(cache: PagedKVCache, cand_keys: torch.Tensor, top_k: int,
                 block_idx: Optional[torch.Tensor] = None, want_scores: bool = False,
                 stream=None):
    """Global selection from the ranks' gathered candidate keys
    [num_lists, batch, Hkv, top_k-1]: the block lists msa_select_topk gives for
    the unsharded sequences."""
    lib = load_library()
    _require_cuda(cand_keys, block_idx)
    nl, batch = cand_keys.shape[0], cand_keys.shape[1]
    if block_idx is None:
        block_idx = torch.empty(batch, cache.num_kv_heads, top_k, dtype=torch.int32,
                                device=cand_keys.device)
    score = (torch.empty(batch, cache.num_kv_heads, top_k, dtype=torch.float32,
                         device=cand_keys.device) if want_scores else None)
    kv = cache.struct()
    _check(lib.msa_select_merge(ctypes.byref(kv), _ptr(cand_keys), nl, top_k, _ptr(block_idx),
                                _ptr(score), _stream(stream)), "msa_select_merge")
    return block_idx, score


def sparse_attn_decode_range(cache: PagedKVCache, q: torch.Tensor, block_idx: torch.Tensor,
                             block_lo: int, block_hi: int, softmax_scale: Optional[float] = None,
                             workspace: Optional[torch.Tensor] = None, stream=None):
    """This rank's attention partial over the selected blocks in [block_lo,
    block_hi): (o_part [batch, Hq, d] fp32 normalised, lse_part [batch, Hq])."""
    lib = load_library()
    _require_cuda(q, block_idx)
    top_k = block_idx.shape[-1]
    scale = 1.0 / math.sqrt(cache.head_dim) if softmax_scale is None else softmax_scale
    o_part = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse_part = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device)
    ws, ws_bytes = _workspace(MSA_OP_DECODE, cache, q.shape[0], 1, top_k, workspace)
    kv = cache.struct()
    _check(lib.msa_sparse_attn_decode_range(ctypes.byref(kv), _ptr(q), _ptr(block_idx), top_k,
                                            int(block_lo), int(block_hi), scale, _ptr(o_part),
                                            _ptr(lse_part), _ptr(ws), ws_bytes, _stream(stream)),
           "msa_sparse_attn_decode_range")
    return o_part, lse_part


def lse_merge(o_parts: torch.Tensor, lse_parts: torch.Tensor, dtype=torch.bfloat16, stream=None):
    """Log-sum-exp merge of partials [P, batch, Hq, d] / [P, batch, Hq] ->
    (out [batch, Hq, d] in dtype, lse [batch, Hq])."""
    lib = load_library()
    _require_cuda(o_parts, lse_parts)
    P, d = o_parts.shape[0], o_parts.shape[-1]
    rows = o_parts[0].numel() // d
    out = torch.empty(o_parts.shape[1:], dtype=dtype, device=o_parts.device)
    lse = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=o_parts.device)
    dt = MSA_DTYPE_BF16 if dtype == torch.bfloat16 else MSA_DTYPE_F32
    _check(lib.msa_lse_merge(_ptr(o_parts), _ptr(lse_parts), P, rows, d, dt, _ptr(out), _ptr(lse),
                             _stream(stream)), "msa_lse_merge")
    return out, lse


def sharded_decode(cache: PagedKVCache, q: torch.Tensor, top_k: int, block_lo: int,
                   block_hi: int, group=None, ops=None):
    """One decode step of context-sharded sequences: this rank holds blocks
    [block_lo, block_hi) of every sequence. Two all-gathers over the process
    group (the ranks' candidate keys; the ranks' attention partials) surround
    the library calls; every rank returns the same (out, lse, block_idx).
    `ops` replaces the four per-rank calls (tests of the exchange on CPU)."""
    import torch.distributed as dist
    ops = ops or {"select": select_topk_range, "merge": select_merge,
                  "attend": sparse_attn_decode_range, "combine": lse_merge}
    world = dist.get_world_size(group)

    def gather(x):  # [world, ...] in rank order
        parts = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(parts, x.contiguous(), group=group)
        return torch.stack(parts)

    keys = ops["select"](cache, q, top_k, block_lo, block_hi)
    block_idx, _ = ops["merge"](cache, gather(keys), top_k)
    o_part, lse_part = ops["attend"](cache, q, block_idx, block_lo, block_hi)
    out, lse = ops["combine"](gather(o_part), gather(lse_part), dtype=q.dtype)
    return out, lse, block_idx


def cu_seqlens(lengths, device="cuda") -> torch.Tensor:
    """[0, l0, l0+l1, ...] as int32 on `device`."""
    c = [0]
    for x in lengths:
        c.append(c[-1] + int(x))
    return torch.tensor(c, dtype=torch.int32, device=device)
