"""Benchmark of the block-sparse GQA attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload prefill_bf16|paged_decode_bf16|decode_1m_bf16|varlen_decode_bf16]

A step is one pass of the whole hot path over one batch of synthetic input:
  prefill workloads : KV append with centroid pooling (msa_build_block_cache),
                      top-k selection (msa_select_topk) and sparse attention
                      (msa_sparse_attn_prefill) over all query rows;
  decode workloads  : append of one token per sequence, decode selection and
                      the stream-K decode attention.
The default workload is the prefill one (batch 1, 32768 tokens, 32/4 heads,
d 128, block 128, top-k 16); the other four workloads are measured in the same
run, one block each in the same JSON line: paged decode ("decode": batch 32,
131072 cached tokens, 32/8 heads, block 64, top-k 32), 1M-context decode
("decode_1m": 256 consecutive steps, each appending one token), varlen decode
("varlen": 64 sequences of 4K-512K tokens) and the tiny fp32 case ("tiny").

Timing: W untimed warm-up steps; the step is then captured in a CUDA graph
(the library never allocates or synchronises) and K replays are timed between
a barrier and torch.cuda.synchronize() on both sides, with CUDA events on the
replay stream, max over ranks. Per-call times come from graphs of each call
alone. The end-to-end figure runs the public Python calls eagerly, with the
step's host-to-device and device-to-host copies inside the timed region. Inputs of every step exceed the 126 MB L2 (prefill: 0.7 GB;
paged decode: ~0.53 GB read per step); the 1M-context decode working set
(~42 MB) does not, so that workload writes a 256 MB buffer between steps.
Under torchrun each rank runs its own replica of the workload (independent
sequences, no collective on the data path): weak scaling.

--impl reference times the CPU fp64 oracle (the reference arm) on a bounded
sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "sparse-attn decode tokens/s + HBM GB/s; prefill tokens/s + tensor-pipe util"


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def profile_traffic(kernel: str, src: str):
    """ncu DRAM bytes per launch recorded in profiles/<kernel>*.md, if the kernel
    source still hashes to the recorded value; else None."""
    return profile_value(kernel, src, "dram_bytes_per_full_launch")


def tensor_pipe(executed_tflops, clocks):
    """Tensor-pipe utilisation of the prefill attention kernel, two ways: the ncu
    counter recorded in its profile (same source hash only), and the executed
    MMA rate of this run against the hardware rate the counter is measured
    against (one M128 N128 K16 bf16 MMA per 64 cycles = 8192 flops/cycle/SM on
    148 SMs at the sampled SM clock)."""
    mhz = clocks.get("sm_mhz") or 1965.0
    hw_tflops = 148 * 8192 * mhz * 1e6 / 1e12
    return {"ncu_active_pct": profile_value("prefill_tc_kernel", "prefill_tc.cu",
                                            "tensor_pipe_active_pct"),
            "ncu_case": "T=16384 capture of the same kernel (profiles/)",
            "hw_rate_tflops": hw_tflops,
            "executed_pct_of_hw_rate": 100.0 * executed_tflops / hw_tflops}


def profile_value(kernel: str, src: str, key: str):
    """A figure `key: value` recorded in profiles/<kernel>*.md, if the kernel
    source still hashes to the recorded value; else None."""
    pdir = os.path.join(ROOT, "profiles")
    sha = hashlib.sha256(open(os.path.join(ROOT, "block_sparse_gqa_mean_b200", "csrc", src),
                              "rb").read()).hexdigest()[:16]
    if not os.path.isdir(pdir):
        return None
    for f in sorted(os.listdir(pdir)):
        if not (f.startswith(kernel) and f.endswith(".md")):
            continue
        vals = {}
        for line in open(os.path.join(pdir, f)):
            if ":" in line and line.strip().startswith(("source_sha256", key)):
                k, v = line.strip().split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
        if vals.get("source_sha256") == sha and key in vals:
            return float(vals[key])
    return None


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"msa_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        smax = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def capture_graph(fn):
    """CUDA graph of fn's launches (the library allocates nothing and never
    synchronises, so every call can be captured)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_graph(g, steps, before=None):
    """Mean device time of one replay (CUDA events on the replay stream).
    `before(i)` runs untimed work (an L2 flush) ahead of replay i."""
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        if before is not None:
            before(i)
        ev[i][0].record(stream)
        g.replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev) / steps


def attended_pairs(T: int, B: int, k: int) -> int:
    """Query-key pairs per head of a full causal prefill: row t sees its own
    block up to t plus k-1 complete past blocks (all of them when fewer)."""
    t = np.arange(T, dtype=np.int64)
    return int(np.minimum(t + 1, (k - 1) * B + (t % B) + 1).sum())


# ---------------------------------------------------------------------------
# prefill workload
# ---------------------------------------------------------------------------
def run_prefill(w, steps, warmup, world):
    import block_sparse_gqa_mean_b200 as msa
    dev = torch.device("cuda")
    T = w.ctx[0]
    p = workloads.paging(w)
    cache = msa.PagedKVCache.allocate(1, p.num_pages, p.max_blocks, w.hq, w.hkv, w.d, w.block,
                                      w.torch_dtype, dev)
    cache.page_table.copy_(p.table.to(dev))
    cache.seq_lens.fill_(T)
    k_new = workloads.keys(w, 0, 0, T, dev).contiguous()
    v_new = workloads.values(w, 0, 0, T, dev).contiguous()
    q = workloads.queries_prefill(w, 0, 0, T, dev).contiguous()
    cu = msa.cu_seqlens([T], dev)
    idx = torch.empty(T, w.hkv, w.top_k, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(T, w.hq, dtype=torch.float32, device=dev)
    ws_sel = torch.empty(max(16, msa.workspace_size(msa.MSA_OP_SELECT, cache, T, T, w.top_k)),
                         dtype=torch.uint8, device=dev)
    ws_att = torch.empty(max(16, msa.workspace_size(msa.MSA_OP_PREFILL, cache, T, T, w.top_k)),
                         dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def do_append():
        msa.build_block_cache(cache, k_new, v_new, cu, T)

    def do_select():
        msa.select_topk(cache, q, w.top_k, cu_q=cu, max_rows_per_seq=T, block_idx=idx,
                        workspace=ws_sel)

    def do_attn():
        msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=T, out=out, lse=lse,
                                workspace=ws_att)

    def step():
        do_append()
        do_select()
        do_attn()

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if cache.device_status() != 0:
        raise RuntimeError(f"device status {cache.device_status():#x}")
    g_step = capture_graph(step)
    g_ops = [capture_graph(f) for f in (do_append, do_select, do_attn)]
    barrier(world)
    torch.cuda.synchronize()
    with Clocks(torch.cuda.current_device()) as clk:
        step_ms = time_graph(g_step, steps)
    barrier(world)
    k_ms = [time_graph(gg, steps) for gg in g_ops]
    total_ms = step_ms * steps

    # executed (union) tile-blocks of the tensor-core schedule, for context: the
    # plan's per-tile union sizes, read back from the call's workspace (entries
    # [units][ecap] int2, then counts [units] int32)
    G = w.group
    TM = 128 // G
    units = ((T + TM - 1) // TM) * w.hkv
    off = units * TM * w.top_k * 8
    union_blocks = int(ws_att[off:off + 4 * units].view(torch.int32).sum().item())

    # end to end through the C ABI from pinned host buffers
    hq_ = q.cpu().pin_memory()
    hk = k_new.cpu().pin_memory()
    hv = v_new.cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k_new), torch.empty_like(v_new)

    def e2e_step():
        dq.copy_(hq_, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        msa.build_block_cache(cache, dk, dv, cu, T)
        msa.select_topk(cache, dq, w.top_k, cu_q=cu, max_rows_per_seq=T, block_idx=idx,
                        workspace=ws_sel)
        msa.sparse_attn_prefill(cache, dq, idx, cu_q=cu, max_rows_per_seq=T, out=out, lse=lse,
                                workspace=ws_att)
        hout.copy_(out, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / steps
    h2d = hq_.numel() * 2 + hk.numel() * 2 + hv.numel() * 2
    d2h = hout.numel() * 2
    status = cache.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status:#x}")
    return {"total_ms": total_ms, "kernel_ms": k_ms, "clocks": clk.summary(),
            "union_blocks": union_blocks, "e2e_ms": e2e_ms, "h2d": h2d, "d2h": d2h,
            "launches_per_step": 5}


# ---------------------------------------------------------------------------
# decode workloads
# ---------------------------------------------------------------------------
def fill_decode_cache(w, dev):
    import block_sparse_gqa_mean_b200 as msa
    p = workloads.paging(w)
    cache = msa.PagedKVCache.allocate(w.batch, p.num_pages, p.max_blocks, w.hq, w.hkv, w.d,
                                      w.block, w.torch_dtype, dev)
    cache.page_table.copy_(p.table.to(dev))
    lens = [0] * w.batch
    chunk = 1 << 16
    for b in range(w.batch):
        for u0 in range(0, w.ctx[b], chunk):
            u1 = min(w.ctx[b], u0 + chunk)
            after = list(lens)
            after[b] = u1
            n = [after[i] - lens[i] for i in range(w.batch)]
            cache.seq_lens.copy_(torch.tensor(after, dtype=torch.int32))
            msa.build_block_cache(cache, workloads.keys(w, b, u0, u1, dev),
                                  workloads.values(w, b, u0, u1, dev), msa.cu_seqlens(n, dev),
                                  max(n))
            lens = after
    torch.cuda.synchronize()
    return cache


def decode_bytes(w, step=0):
    """Algorithmic HBM bytes of one decode step: the centroid scan of every
    complete past block, the K/V rows of the selected blocks (own block up to
    the new token), q in / out, the appended K/V row and its centroid."""
    tot = 0
    for b in range(w.batch):
        L = w.ctx[b] + step + 1
        own = (L - 1) // w.block
        cand = own
        take = min(w.top_k - 1, cand)
        keys = take * w.block + (L - own * w.block)
        tot += w.hkv * (cand * w.d * 4 + keys * w.d * 2 * 2)
        tot += 2 * w.hq * w.d * 2 + 2 * w.hkv * w.d * 2 + w.hkv * w.d * 4
    return tot


def run_decode(w, steps, warmup, world, flush_l2):
    import block_sparse_gqa_mean_b200 as msa
    dev = torch.device("cuda")
    cache = fill_decode_cache(w, dev)
    after = [w.ctx[b] + 1 for b in range(w.batch)]
    cache.seq_lens.copy_(torch.tensor(after, dtype=torch.int32))
    kn, vn = workloads.new_tokens(w, 0, dev)
    q = workloads.queries_decode(w, 0, dev).contiguous()
    cu = msa.cu_seqlens([1] * w.batch, dev)
    idx = torch.empty(w.batch, w.hkv, w.top_k, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(w.batch, w.hq, dtype=torch.float32, device=dev)
    ws_sel = torch.empty(max(16, msa.workspace_size(msa.MSA_OP_SELECT, cache, w.batch, 1, w.top_k)),
                         dtype=torch.uint8, device=dev)
    ws_dec = torch.empty(max(16, msa.workspace_size(msa.MSA_OP_DECODE, cache, w.batch, 1, w.top_k)),
                         dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush_l2 else None
    stream = torch.cuda.current_stream()

    def do_append():
        msa.build_block_cache(cache, kn, vn, cu, 1)

    def do_select():
        msa.select_topk(cache, q, w.top_k, block_idx=idx, workspace=ws_sel)

    def do_attn():
        msa.sparse_attn_decode(cache, q, idx, out=out, lse=lse, workspace=ws_dec)

    def step():
        do_append()
        do_select()
        do_attn()

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    g_step = capture_graph(step)
    g_ops = [capture_graph(f) for f in (do_append, do_select, do_attn)]
    flush_fn = (lambda i: flush.fill_(i & 0xFF)) if flush is not None else None
    barrier(world)
    torch.cuda.synchronize()
    with Clocks(torch.cuda.current_device()) as clk:
        step_ms = time_graph(g_step, steps, flush_fn)
    barrier(world)
    k_ms = [time_graph(gg, steps, flush_fn) for gg in g_ops]
    per_step = [step_ms]

    # end to end: q and the new K/V rows from pinned host memory, out back to host
    hq_, hk, hv = q.cpu().pin_memory(), kn.cpu().pin_memory(), vn.cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(kn), torch.empty_like(vn)

    def e2e_step():
        dq.copy_(hq_, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        msa.build_block_cache(cache, dk, dv, cu, 1)
        msa.select_topk(cache, dq, w.top_k, block_idx=idx, workspace=ws_sel)
        msa.sparse_attn_decode(cache, dq, idx, out=out, lse=lse, workspace=ws_dec)
        hout.copy_(out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e2e = []
    for _ in range(steps):
        if flush is not None:
            flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b.record(stream)
        e2e.append((a, b))
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e) / steps
    status = cache.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status:#x}")
    return {"step_ms": per_step[0], "kernel_ms": k_ms, "clocks": clk.summary(),
            "e2e_ms": e2e_ms, "h2d": (hq_.numel() + hk.numel() + hv.numel()) * 2,
            "d2h": hout.numel() * 2, "launches_per_step": 1 + 2 + 1}


def run_decode_steps(w, world):
    """Consecutive decode steps (the 1M-context workload): step s sets the
    length to ctx + s + 1, appends token ctx + s, selects with step s's query
    and attends. One CUDA graph per step (each holds its own input and output
    pointers and length), replayed in order; an untimed 256 MB write flushes
    L2 before every step (the step's ~42 MB would otherwise stay in L2)."""
    import block_sparse_gqa_mean_b200 as msa
    dev = torch.device("cuda")
    cache = fill_decode_cache(w, dev)
    S, nb = w.steps, w.batch
    lens = torch.tensor([[w.ctx[b] + s + 1 for b in range(nb)] for s in range(S)],
                        dtype=torch.int32, device=dev)
    toks = [workloads.new_tokens(w, s, dev) for s in range(S)]
    k_all = torch.stack([t[0] for t in toks]).contiguous()         # [S, batch, hkv, d]
    v_all = torch.stack([t[1] for t in toks]).contiguous()
    q_all = torch.stack([workloads.queries_decode(w, s, dev) for s in range(S)]).contiguous()
    out_all = torch.empty_like(q_all)
    lse_all = torch.empty(S, nb, w.hq, dtype=torch.float32, device=dev)
    cu = msa.cu_seqlens([1] * nb, dev)
    idx = torch.empty(nb, w.hkv, w.top_k, dtype=torch.int32, device=dev)
    ws_sel = torch.empty(max(16, msa.workspace_size(msa.MSA_OP_SELECT, cache, nb, 1, w.top_k)),
                         dtype=torch.uint8, device=dev)
    ws_dec = torch.empty(max(16, msa.workspace_size(msa.MSA_OP_DECODE, cache, nb, 1, w.top_k)),
                         dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def calls(s):
        def do_len():
            cache.seq_lens.copy_(lens[s])       # the caller advances the lengths
        def do_append():
            msa.build_block_cache(cache, k_all[s], v_all[s], cu, 1)
        def do_select():
            msa.select_topk(cache, q_all[s], w.top_k, block_idx=idx, workspace=ws_sel)
        def do_attn():
            msa.sparse_attn_decode(cache, q_all[s], idx, out=out_all[s], lse=lse_all[s],
                                   workspace=ws_dec)
        return do_len, do_append, do_select, do_attn

    def step_fn(s):
        fs = calls(s)
        return lambda: [f() for f in fs]

    graphs = [capture_graph(step_fn(s)) for s in range(S)]   # also runs each step once, in order
    for g in graphs:                                           # warm-up: the whole run once more
        g.replay()
    torch.cuda.synchronize()
    if cache.device_status() != 0:
        raise RuntimeError(f"device status {cache.device_status():#x}")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(S)]
    barrier(world)
    torch.cuda.synchronize()
    with Clocks(torch.cuda.current_device()) as clk:
        for s in range(S):
            flush.fill_(s & 0xFF)
            ev[s][0].record(stream)
            graphs[s].replay()
            ev[s][1].record(stream)
        torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    # per-call times on the last step (re-appending its token is idempotent)
    fl, fa, fs_, ft = calls(S - 1)
    g_ops = [capture_graph(lambda: (fl(), fa())), capture_graph(fs_), capture_graph(ft)]
    k_ms = [time_graph(gg, 20, lambda i: flush.fill_(i & 0xFF)) for gg in g_ops]

    # end to end: every step's q and new K/V rows from pinned host memory, its
    # output back to the host, eager calls
    hq_, hk, hv = q_all.cpu().pin_memory(), k_all.cpu().pin_memory(), v_all.cpu().pin_memory()
    hout = torch.empty(out_all.shape, dtype=out_all.dtype).pin_memory()
    dq, dk, dv = torch.empty_like(q_all[0]), torch.empty_like(k_all[0]), torch.empty_like(v_all[0])
    dout = torch.empty_like(out_all[0])
    dlse = torch.empty_like(lse_all[0])
    e2e = []
    for s in range(S):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dq.copy_(hq_[s], non_blocking=True)
        dk.copy_(hk[s], non_blocking=True)
        dv.copy_(hv[s], non_blocking=True)
        cache.seq_lens.copy_(lens[s])
        msa.build_block_cache(cache, dk, dv, cu, 1)
        msa.select_topk(cache, dq, w.top_k, block_idx=idx, workspace=ws_sel)
        msa.sparse_attn_decode(cache, dq, idx, out=dout, lse=dlse, workspace=ws_dec)
        hout[s].copy_(dout, non_blocking=True)
        b.record(stream)
        e2e.append((a, b))
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e) / S
    if not torch.equal(hout.view(torch.int16), out_all.cpu().view(torch.int16)):
        raise RuntimeError("end-to-end outputs differ from the graph replays")
    status = cache.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status:#x}")
    return {"step_ms": sum(step_ms) / S, "step_ms_first_last": [step_ms[0], step_ms[-1]],
            "kernel_ms": k_ms, "clocks": clk.summary(), "e2e_ms": e2e_ms,
            "h2d": (hq_[0].numel() + hk[0].numel() + hv[0].numel()) * 2,
            "d2h": hout[0].numel() * 2, "launches_per_step": 1 + 2 + 1, "steps": S}


TOKEN_HEADS = 32      # indexer heads ("Sparse Attention + Linear Backbones", 5.3: 32 x 128)
TOKEN_TOP_K = 2048    # kept positions per query (same section)


def index_pages(w, p, lens, dev):
    """Indexer keys of every sequence, one row per position, written into pages
    of the cache's page table: [num_pages, block, d]."""
    ki = torch.zeros(p.num_pages, w.block, w.d, dtype=w.torch_dtype, device=dev)
    for b in range(w.batch):
        L = lens[b]
        nblk = -(-L // w.block)
        rows = torch.zeros(nblk * w.block, w.d, dtype=w.torch_dtype, device=dev)
        rows[:L] = workloads.indexer_keys(w, b, 0, L, dev)
        ki[p.table[b, :nblk].long().to(dev)] = rows.view(nblk, w.block, w.d)
    return ki


def token_bytes(w, k):
    """Algorithmic HBM bytes of one token-variant decode step: the indexer key of
    every earlier position, the kept positions' K and V rows, q, out, the
    indexer query, and the appended K/V row, its centroid and its indexer key."""
    tot = 0
    for b in range(w.batch):
        L = w.ctx[b] + 1
        tot += (L - 1) * w.d * 2 + min(k, L) * w.hkv * w.d * 2 * 2
        tot += 2 * w.hq * w.d * 2 + TOKEN_HEADS * w.d * 2
        tot += 2 * w.hkv * w.d * 2 + w.hkv * w.d * 4 + w.d * 2
    return tot


def run_tokens(w, steps, world):
    """The token-granular variant on the paged-decode context: append one token
    per sequence (with its indexer key), the indexer scores every earlier
    position and keeps the top-K, then attention over the kept positions."""
    import block_sparse_gqa_mean_b200 as msa
    dev = torch.device("cuda")
    cache = fill_decode_cache(w, dev)
    after = [w.ctx[b] + 1 for b in range(w.batch)]
    cache.seq_lens.copy_(torch.tensor(after, dtype=torch.int32))
    p = workloads.paging(w)
    ki = index_pages(w, p, after, dev)
    kn, vn = workloads.new_tokens(w, 0, dev)
    q = workloads.queries_decode(w, 0, dev).contiguous()
    qi = workloads.indexer_queries(w, 0, TOKEN_HEADS, dev).contiguous()
    # the appended token's indexer-key row: where it lives in the pages
    last = torch.tensor([[int(p.table[b, (L - 1) // w.block]), (L - 1) % w.block]
                         for b, L in enumerate(after)], dtype=torch.long, device=dev)
    ki_new = torch.stack([ki[last[b, 0], last[b, 1]] for b in range(w.batch)]).contiguous()
    cu = msa.cu_seqlens([1] * w.batch, dev)
    tok = torch.empty(w.batch, TOKEN_TOP_K, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(w.batch, w.hq, dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, msa.workspace_size(msa.MSA_OP_SELECT_TOKENS, cache, w.batch, 1,
                                                TOKEN_TOP_K)), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def do_append():
        msa.build_block_cache(cache, kn, vn, cu, 1)
        ki[last[:, 0], last[:, 1]] = ki_new          # the caller writes the indexer key

    def do_select():
        msa.select_tokens(cache, ki, qi, TOKEN_TOP_K, tok_idx=tok, workspace=ws)

    def do_attn():
        msa.sparse_attn_decode_tokens(cache, q, tok, out=out, lse=lse)

    def step():
        do_append()
        do_select()
        do_attn()

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    g_step = capture_graph(step)
    g_ops = [capture_graph(f) for f in (do_append, do_select, do_attn)]
    barrier(world)
    torch.cuda.synchronize()
    with Clocks(torch.cuda.current_device()) as clk:
        step_ms = time_graph(g_step, steps)
    k_ms = [time_graph(gg, steps) for gg in g_ops]
    hq_, hqi = q.cpu().pin_memory(), qi.cpu().pin_memory()
    hk, hv, hki = kn.cpu().pin_memory(), vn.cpu().pin_memory(), ki_new.cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dq, dqi = torch.empty_like(q), torch.empty_like(qi)
    dk, dv, dki = torch.empty_like(kn), torch.empty_like(vn), torch.empty_like(ki_new)
    e2e = []
    for _ in range(steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for d_, h_ in ((dq, hq_), (dqi, hqi), (dk, hk), (dv, hv), (dki, hki)):
            d_.copy_(h_, non_blocking=True)
        msa.build_block_cache(cache, dk, dv, cu, 1)
        ki[last[:, 0], last[:, 1]] = dki
        msa.select_tokens(cache, ki, dqi, TOKEN_TOP_K, tok_idx=tok, workspace=ws)
        msa.sparse_attn_decode_tokens(cache, dq, tok, out=out, lse=lse)
        hout.copy_(out, non_blocking=True)
        b.record(stream)
        e2e.append((a, b))
    torch.cuda.synchronize()
    if cache.device_status() != 0:
        raise RuntimeError(f"device status {cache.device_status():#x}")
    h2d = sum(x.numel() * x.element_size() for x in (hq_, hqi, hk, hv, hki))
    return {"step_ms": step_ms, "kernel_ms": k_ms, "clocks": clk.summary(),
            "e2e_ms": sum(a.elapsed_time(b) for a, b in e2e) / steps, "h2d": h2d,
            "d2h": hout.numel() * 2, "launches_per_step": 1 + 2 + 1}


def tokens_block(w, args, world, pk):
    """Block of the token-granular variant (decode form) on the paged-decode context."""
    r = run_tokens(w, args.steps, world)
    ms = max_over_ranks(r["step_ms"], world)
    nbytes = token_bytes(w, TOKEN_TOP_K)
    sel_b = sum((w.ctx[b]) * w.d * 2 + TOKEN_HEADS * w.d * 2 for b in range(w.batch))
    att_b = sum(min(TOKEN_TOP_K, w.ctx[b] + 1) * w.hkv * w.d * 4 + 2 * w.hq * w.d * 2
                for b in range(w.batch))
    sel_ms, att_ms = r["kernel_ms"][1], r["kernel_ms"][2]
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": w.name + " (token-granular indexer)", "value": w.batch * world / (ms * 1e-3),
            "unit": "tokens/s", "ms_per_step": ms, "indexer_heads": TOKEN_HEADS,
            "top_k_tokens": TOKEN_TOP_K,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": None,
                         "peak_source": f"{pk['source']} HBM copy",
                         "scope": "whole decode step (append + indexer selection + attention)",
                         "algorithmic_bytes_per_step": nbytes,
                         "calls": {
                             "select_tokens": {"bytes": sel_b, "ms": sel_ms,
                                               "achieved_gbs": sel_b / (sel_ms * 1e-3) / 1e9},
                             "sparse_attn_decode_tokens": {
                                 "bytes": att_b, "ms": att_ms,
                                 "achieved_gbs": att_b / (att_ms * 1e-3) / 1e9}}},
            "kernels_ms": {"append": r["kernel_ms"][0], "select_tokens": sel_ms,
                           "sparse_attn_decode_tokens": att_ms},
            "e2e": {"value": w.batch * world / (r["e2e_ms"] * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
            "clocks": r["clocks"], "gpu_launches": r["launches_per_step"] * args.steps,
            "l2": "step reads > 126 MB L2, no flush"}


def oracle_tokens_sample(w, device="cpu"):
    """Oracle of the token variant on sequence 0's decode step (inputs drawn on
    `device`, outside the timed region). Returns (sequences, seconds, threads)."""
    import oracle
    L = w.ctx[0] + 1
    K = workloads.keys(w, 0, 0, L, device).cpu()
    V = workloads.values(w, 0, 0, L, device).cpu()
    KI = workloads.indexer_keys(w, 0, 0, L, device).cpu()
    Q = workloads.queries_decode(w, 0, seqs=[0])
    QI = workloads.indexer_queries(w, 0, TOKEN_HEADS)[:1]
    pos = np.array([L - 1])
    t = time.perf_counter()
    S = oracle.token_scores(QI, KI, pos)
    idx, _ = oracle.token_select(S, pos, TOKEN_TOP_K)
    oracle.attend_tokens(Q, K, V, pos, idx, w.softmax_scale)
    return 1, time.perf_counter() - t, 1


def run_tiny(w, steps, world):
    """The tiny fp32 workload: prefill of all 1024 rows (append, select,
    attention; fp32 SIMT kernels), then the decode step that appends token
    1023 onto 1023 cached tokens and attends."""
    import block_sparse_gqa_mean_b200 as msa
    dev = torch.device("cuda")
    T = w.ctx[0]
    p = workloads.paging(w)
    cache = msa.PagedKVCache.allocate(1, p.num_pages, p.max_blocks, w.hq, w.hkv, w.d, w.block,
                                      w.torch_dtype, dev)
    cache.page_table.copy_(p.table.to(dev))
    K = workloads.keys(w, 0, 0, T, dev).contiguous()
    V = workloads.values(w, 0, 0, T, dev).contiguous()
    q = workloads.queries_prefill(w, 0, 0, T, dev).contiguous()
    cu = msa.cu_seqlens([T], dev)
    cu1 = msa.cu_seqlens([1], dev)
    idx = torch.empty(T, w.hkv, w.top_k, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(T, w.hq, dtype=torch.float32, device=dev)
    didx = torch.empty(1, w.hkv, w.top_k, dtype=torch.int32, device=dev)
    dout = torch.empty_like(q[:1])
    dlse = torch.empty(1, w.hq, dtype=torch.float32, device=dev)
    lens_p = torch.tensor([T], dtype=torch.int32, device=dev)
    qd = q[T - 1:].contiguous()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def prefill():
        cache.seq_lens.copy_(lens_p)
        msa.build_block_cache(cache, K, V, cu, T)
        msa.select_topk(cache, q, w.top_k, cu_q=cu, max_rows_per_seq=T, block_idx=idx)
        msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=T, out=out, lse=lse)

    def decode():
        cache.seq_lens.copy_(lens_p)                 # token 1023 appended onto 1023 cached
        msa.build_block_cache(cache, K[T - 1:], V[T - 1:], cu1, 1)
        msa.select_topk(cache, qd, w.top_k, block_idx=didx)
        msa.sparse_attn_decode(cache, qd, didx, out=dout, lse=dlse)

    g_p, g_d = capture_graph(prefill), capture_graph(decode)
    for _ in range(3):
        g_p.replay()
        g_d.replay()
    torch.cuda.synchronize()
    flush_fn = lambda i: flush.fill_(i & 0xFF)
    barrier(world)
    with Clocks(torch.cuda.current_device()) as clk:
        p_ms = time_graph(g_p, steps, flush_fn)
        d_ms = time_graph(g_d, steps, flush_fn)
    if (dout - out[T - 1:]).abs().max().item() > 1e-6:
        raise RuntimeError("tiny decode differs from prefill row 1023")
    hq_, hk, hv = q.cpu().pin_memory(), K.cpu().pin_memory(), V.cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(K), torch.empty_like(V)
    stream = torch.cuda.current_stream()
    e2e = []
    for _ in range(steps):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dq.copy_(hq_, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        cache.seq_lens.copy_(lens_p)
        msa.build_block_cache(cache, dk, dv, cu, T)
        msa.select_topk(cache, dq, w.top_k, cu_q=cu, max_rows_per_seq=T, block_idx=idx)
        msa.sparse_attn_prefill(cache, dq, idx, cu_q=cu, max_rows_per_seq=T, out=out, lse=lse)
        hout.copy_(out, non_blocking=True)
        b.record(stream)
        e2e.append((a, b))
    torch.cuda.synchronize()
    if cache.device_status() != 0:
        raise RuntimeError(f"device status {cache.device_status():#x}")
    return {"prefill_ms": p_ms, "decode_ms": d_ms, "clocks": clk.summary(),
            "e2e_ms": sum(a.elapsed_time(b) for a, b in e2e) / steps,
            "h2d": (hq_.numel() + hk.numel() + hv.numel()) * 4, "d2h": hout.numel() * 4,
            "launches_per_step": 3}


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------
def oracle_prefill_sample(w, rows: int):
    """Oracle on a bounded sample: the block cache of the whole sequence plus
    `rows` query rows spread over the sequence. Returns (rows, seconds, threads)."""
    import oracle
    T = w.ctx[0]
    K = workloads.keys(w, 0, 0, T)
    V = workloads.values(w, 0, 0, T)
    pos = np.linspace(0, T - 1, rows).astype(np.int64)
    Q = torch.cat([workloads.queries_prefill(w, 0, int(r), int(r) + 1) for r in pos])
    t = time.perf_counter()
    oracle.forward(Q, K, V, pos, w.block, w.top_k, w.softmax_scale)
    return rows, time.perf_counter() - t, oracle.num_threads()


def oracle_decode_sample(w, seqs, device="cpu"):
    """Oracle on the decode step of the listed sequences (the inputs are drawn
    on `device`, outside the timed region; the oracle runs on the host).
    Returns (sequences, seconds, threads)."""
    import oracle
    secs, n = 0.0, 0
    for b in seqs:
        L = w.ctx[b] + 1
        K = workloads.keys(w, b, 0, L, device).cpu()
        V = workloads.values(w, b, 0, L, device).cpu()
        Q = workloads.queries_decode(w, 0, seqs=[b])
        t = time.perf_counter()
        oracle.forward(Q, K, V, np.array([L - 1]), w.block, w.top_k, w.softmax_scale)
        secs += time.perf_counter() - t
        n += 1
    return n, secs, oracle.num_threads()


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="prefill_bf16", choices=list(workloads.ALL))
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the blocks of the other workloads")
    ap.add_argument("--blocks", default="decode,decode_1m,varlen,tiny,tokens",
                    help="workload blocks measured after the prefill headline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--oracle-rows", type=int, default=256)
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override the prefill length (profiling of a smaller case)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the decode batch (profiling of a smaller case)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup()
    w = workloads.ALL[args.workload]()
    if args.seq_len and w.kind == "prefill":
        w = workloads.ALL[args.workload](ctx=(args.seq_len,))
    if args.batch and w.kind == "decode" and w.name != "decode_1m_bf16":
        w = workloads.ALL[args.workload](batch=args.batch)
    pk = peaks()

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(w, args)))
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py --impl native needs a CUDA device")
    import block_sparse_gqa_mean_b200 as msa
    msa.load_library()

    res = {}
    if w.kind == "prefill":
        r = run_prefill(w, args.steps, args.warmup, world)
        ms = max_over_ranks(r["total_ms"] / args.steps, world)
        T = w.ctx[0]
        pairs = attended_pairs(T, w.block, w.top_k) * w.hq
        flops = 4.0 * w.d * pairs
        attn_ms = max_over_ranks(r["kernel_ms"][2], world)
        achieved = flops / (attn_ms * 1e-3) / 1e12
        executed = r["union_blocks"] * 128 * w.block * w.d * 4.0
        traffic = profile_traffic("prefill_tc_kernel", "prefill_tc.cu")
        res.update({
            "metric": METRIC, "value": T * world / (ms * 1e-3), "unit": "tokens/s",
            "ms_per_step": ms,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                         "traffic": traffic,
                         "peak_source": f"{pk['source']} bf16 (burst cuBLAS)",
                         "kernel": "msa_sparse_attn_prefill (cluster + plan + prefill_tc_kernel)",
                         "algorithmic_flops_per_launch": flops,
                         "executed_mma_flops_per_launch": executed,
                         "executed_tflops": executed / (attn_ms * 1e-3) / 1e12,
                         "tensor_pipe": tensor_pipe(executed / (attn_ms * 1e-3) / 1e12,
                                                    r["clocks"])},
            "kernels_ms": {"build_block_cache": r["kernel_ms"][0], "select_topk": r["kernel_ms"][1],
                           "sparse_attn_prefill": r["kernel_ms"][2]},
            "e2e": {"value": T * world / (max_over_ranks(r["e2e_ms"], world) * 1e-3),
                    "unit": "tokens/s", "h2d_bytes_per_step": r["h2d"],
                    "d2h_bytes_per_step": r["d2h"]},
            "gpu_launches": r["launches_per_step"] * args.steps,
            "clocks": r["clocks"],
            "config": workload_config(w),
        })
        if not args.no_decode and world == 1:
            res.update(extra_blocks(args, world, pk))
    else:
        res.update(decode_main(w, args, world, pk))

    res.update({"n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16 in, fp32 accumulate" if w.dtype == "bf16" else "f32",
                "data": "synthetic (seeded generator, planted relevant blocks)"})
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, args)
    if rank == 0:
        print(json.dumps(res))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def decode_call_bytes(w, step=0):
    """Algorithmic HBM bytes of the selection call (centroid scan, q) and of the
    attention call (K/V rows of the selected blocks, q, out)."""
    sel = att = 0
    for b in range(w.batch):
        L = w.ctx[b] + step + 1
        own = (L - 1) // w.block
        take = min(w.top_k - 1, own)
        keys = take * w.block + (L - own * w.block)
        sel += w.hkv * own * w.d * 4 + w.hq * w.d * 2
        att += w.hkv * keys * w.d * 2 * 2 + 2 * w.hq * w.d * 2
    return sel, att


def decode_block(w, args, world, pk):
    flush = decode_flush(w)
    r = run_decode(w, args.steps, args.warmup, world, flush)
    ms = max_over_ranks(r["step_ms"], world)
    nbytes = decode_bytes(w)
    sel_b, att_b = decode_call_bytes(w)
    sel_ms = max_over_ranks(r["kernel_ms"][1], world)
    att_ms = max_over_ranks(r["kernel_ms"][2], world)
    # DRAM bytes of the two streaming kernels from their ncu summaries (paged
    # decode workload only), None once either source has changed
    traffic = None
    if w.name == "paged_decode_bf16" and w.batch == 32:
        t1 = profile_traffic("select_decode_pass1", "select.cu")
        t2 = profile_traffic("decode_streamk_kernel", "decode_splitk.cu")
        traffic = t1 + t2 if t1 is not None and t2 is not None else None
    return {"workload": w.name, "value": w.batch * world / (ms * 1e-3), "unit": "tokens/s",
            "ms_per_step": ms, "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
            "roofline": {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9,
                         "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                         "traffic": traffic,
                         "traffic_scope": "select_decode_pass1 + decode_streamk_kernel DRAM bytes",
                         "peak_source": f"{pk['source']} HBM copy",
                         "scope": "whole decode step (append+select+attention)",
                         "algorithmic_bytes_per_step": nbytes,
                         "calls": {
                             "select_topk": {"bytes": sel_b, "ms": sel_ms,
                                             "achieved_gbs": sel_b / (sel_ms * 1e-3) / 1e9},
                             "sparse_attn_decode": {"bytes": att_b, "ms": att_ms,
                                                    "achieved_gbs": att_b / (att_ms * 1e-3) / 1e9}}},
            "kernels_ms": {"build_block_cache": r["kernel_ms"][0], "select_topk": sel_ms,
                           "sparse_attn_decode": att_ms},
            "e2e": {"value": w.batch * world / (r["e2e_ms"] * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
            "clocks": r["clocks"], "gpu_launches": r["launches_per_step"] * args.steps,
            "l2": "256 MB write between steps" if flush else "step reads > 126 MB L2, no flush"}


def extra_blocks(args, world, pk):
    """The other four workloads, measured in the same run, one block each."""
    out = {}
    for key in [b for b in args.blocks.split(",") if b]:
        torch.cuda.empty_cache()
        if key == "decode":
            w = workloads.paged_decode_bf16()
            out[key] = decode_block(w, args, world, pk)
        elif key == "varlen":
            w = workloads.varlen_decode_bf16()
            out[key] = decode_block(w, args, world, pk)
        elif key == "decode_1m":
            w = workloads.decode_1m_bf16()
            out[key] = steps_block(w, args, world, pk)
        elif key == "tiny":
            w = workloads.tiny_f32()
            out[key] = tiny_block(w, args, world, pk)
        elif key == "tokens":
            w = workloads.paged_decode_bf16()
            out[key] = tokens_block(w, args, world, pk)
            if not args.no_cpu_baseline and world == 1:
                n, secs, thr = oracle_tokens_sample(w, "cuda")
                out[key]["cpu_baseline"] = {
                    "value": n / secs, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                    "sample": f"sequence 0's decode step ({w.ctx[0] + 1} positions): indexer "
                              f"scores, top-{TOKEN_TOP_K}, attention; numpy fp64"}
            out[key]["config"] = workload_config(w)
            continue
        else:
            raise SystemExit(f"unknown block {key}")
        if not args.no_cpu_baseline and world == 1:
            out[key]["cpu_baseline"] = cpu_baseline(w, args)
        out[key]["config"] = workload_config(w)
    return out


def steps_block(w, args, world, pk):
    """Block of the consecutive-step decode workload (1M context, 256 steps)."""
    r = run_decode_steps(w, world)
    ms = max_over_ranks(r["step_ms"], world)
    nbytes = sum(decode_bytes(w, s) for s in range(w.steps)) / w.steps
    sel_b, att_b = decode_call_bytes(w, w.steps - 1)
    sel_ms, att_ms = r["kernel_ms"][1], r["kernel_ms"][2]
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": w.name, "value": w.batch * world / (ms * 1e-3), "unit": "tokens/s",
            "ms_per_step": ms, "steps": r["steps"], "step_ms_first_last": r["step_ms_first_last"],
            "hbm_gbs": gbs,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": None,
                         "peak_source": f"{pk['source']} HBM copy",
                         "scope": "whole decode step (append+select+attention), mean of the "
                                  f"{w.steps} consecutive steps",
                         "algorithmic_bytes_per_step": nbytes,
                         "calls": {
                             "select_topk": {"bytes": sel_b, "ms": sel_ms,
                                             "achieved_gbs": sel_b / (sel_ms * 1e-3) / 1e9},
                             "sparse_attn_decode": {"bytes": att_b, "ms": att_ms,
                                                    "achieved_gbs": att_b / (att_ms * 1e-3) / 1e9}}},
            "kernels_ms": {"build_block_cache": r["kernel_ms"][0], "select_topk": sel_ms,
                           "sparse_attn_decode": att_ms},
            "e2e": {"value": w.batch * world / (r["e2e_ms"] * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
            "clocks": r["clocks"], "gpu_launches": r["launches_per_step"] * r["steps"],
            "l2": "256 MB write before every step"}


def tiny_block(w, args, world, pk):
    """Block of the tiny fp32 workload (correctness-sized; fp32 SIMT kernels)."""
    r = run_tiny(w, args.steps, world)
    T = w.ctx[0]
    flops = 4.0 * w.d * attended_pairs(T, w.block, w.top_k) * w.hq
    ms = max_over_ranks(r["prefill_ms"], world)
    # fp32 FMA peak from the unit counts: 148 SMs x 128 lanes x 2 flops x clock
    clk = r["clocks"].get("sm_mhz") or 1965.0
    peak = 148 * 128 * 2 * clk * 1e6 / 1e12
    achieved = flops / (ms * 1e-3) / 1e12
    return {"workload": w.name, "value": T * world / (ms * 1e-3), "unit": "tokens/s",
            "ms_per_step": ms, "decode_ms": r["decode_ms"],
            "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None,
                         "peak_source": "fp32 FMA lanes x clock (148 x 128 x 2 x sampled SM MHz)",
                         "scope": "whole prefill step (append+select+attention; 1024 rows, "
                                  "latency-bound at this size)",
                         "algorithmic_flops_per_step": flops},
            "e2e": {"value": T * world / (r["e2e_ms"] * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
            "clocks": r["clocks"], "gpu_launches": r["launches_per_step"] * args.steps,
            "l2": "256 MB write between steps"}


def decode_main(w, args, world, pk):
    d = steps_block(w, args, world, pk) if w.steps > 1 else decode_block(w, args, world, pk)
    return {"metric": METRIC, "value": d["value"], "unit": "tokens/s", "ms_per_step": d["ms_per_step"],
            "roofline": d["roofline"], "kernels_ms": d["kernels_ms"], "e2e": d["e2e"],
            "clocks": d["clocks"], "gpu_launches": d["gpu_launches"],
            "config": workload_config(w)}


def decode_flush(w):
    """The 1M-context step reads ~41 MB, inside L2: flush it between steps."""
    return w.name == "decode_1m_bf16"


def workload_config(w):
    """The config object of the JSON line (the same for both arms)."""
    c = {"workload": w.name, "batch": w.batch, "q_heads": w.hq, "kv_heads": w.hkv,
         "head_dim": w.d, "block": w.block, "top_k": w.top_k}
    if w.kind == "prefill":
        c.update({"seq_len": w.ctx[0],
                  "l2": ("256 MB write between steps" if w.name == "tiny_f32"
                         else "inputs 0.7 GB per step > 126 MB L2, no flush")})
    else:
        c.update({"context_mean": float(np.mean(w.ctx)),
                  "l2": ("256 MB write between steps" if decode_flush(w)
                         else "step reads > 126 MB L2, no flush")})
    return c


def cpu_baseline(w, args):
    if w.kind == "prefill":
        n, secs, thr = oracle_prefill_sample(w, args.oracle_rows)
        return {"value": n / secs, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                "sample": f"{n} query rows spread over the {w.ctx[0]}-token sequence, plus the "
                          f"block cache of the whole sequence, fp64, OpenMP"}
    seqs = sample_seqs(w)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    n, secs, thr = oracle_decode_sample(w, seqs, dev)
    return {"value": n / secs, "unit": "tokens/s", "cores": thr, "kind": "oracle",
            "sample": f"{n} of {w.batch} sequences' decode step (lengths "
                      f"{[w.ctx[b] + 1 for b in seqs]}: block cache of the whole context + "
                      f"selection + attention), fp64, OpenMP"}


def sample_seqs(w):
    """Sequences of the bounded CPU sample of a decode workload: the first two,
    or for varied lengths the one closest to the mean length."""
    if len(set(w.ctx)) > 1:
        mean = float(np.mean(w.ctx))
        return [int(np.argmin([abs(L - mean) for L in w.ctx]))]
    return list(range(min(w.batch, 2 if w.ctx[0] <= (1 << 17) else 1)))


def reference_arm(w, args):
    """The CPU oracle timed as the reference arm: each step is a bounded sample."""
    steps = []
    for i in range(args.warmup + args.steps):
        if w.kind == "prefill":
            n, secs, thr = oracle_prefill_sample(w, max(8, args.oracle_rows // 4))
        else:
            n, secs, thr = oracle_decode_sample(w, sample_seqs(w)[:1])
        if i >= args.warmup:
            steps.append((n, secs))
    n = sum(s[0] for s in steps)
    secs = sum(s[1] for s in steps)
    value = n / secs
    sample = (f"{steps[0][0]} query rows of the {w.ctx[0]}-token prefill per step"
              if w.kind == "prefill" else "1 sequence's decode step per step")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / len(steps), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


if __name__ == "__main__":
    main()
