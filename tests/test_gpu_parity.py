"""GPU-vs-oracle parity on seeded inputs, through the C ABI (Python binding).

Sizes here are small enough for the fp64 oracle to finish in seconds while
spanning several query tiles, several blocks and ragged tails. Every input is
drawn by the `workloads` generator on the GPU and independently regenerated on
the CPU for the oracle (the generator is bit-identical across devices, which
test_generator_bits_match checks).
"""
import numpy as np
import pytest
import torch

import block_sparse_gqa_mean_b200 as msa
import oracle
import workloads
from msa_harness import (append, check_index_invariants, check_selection, compare, fill_context,
                         new_cache, oracle_rows, read_pages)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_library_loads_on_gpu():
    assert torch.cuda.is_available()
    assert msa.load_library().msa_version() >= 1000


def test_generator_bits_match():
    w = workloads.prefill_bf16()
    for (u0, u1) in [(0, 300), (12345, 12400)]:
        a = workloads.keys(w, 0, u0, u1, DEV).cpu()
        b = workloads.keys(w, 0, u0, u1, "cpu")
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        qa = workloads.queries_prefill(w, 0, u0, u1, DEV).cpu()
        qb = workloads.queries_prefill(w, 0, u0, u1, "cpu")
        assert torch.equal(qa.view(torch.int16), qb.view(torch.int16))
    wt = workloads.tiny_f32()
    assert torch.equal(workloads.keys(wt, 0, 0, 1024, DEV).cpu(), workloads.keys(wt, 0, 0, 1024))


# ---------------------------------------------------------------------------
# block cache
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_append_pool_matches_oracle_and_rebuild(dtype):
    d, B = (128, 128) if dtype == "bf16" else (64, 64)
    w = workloads.paged_decode_bf16(batch=3, ctx=(1000, 257, 3000), block=B, d=d, dtype=dtype,
                                    hq=8, hkv=2, steps=0)
    p = workloads.paging(w)
    # one-shot build
    c1 = new_cache(w, p)
    append(c1, w, [0] * 3, list(w.ctx))
    # ragged multi-call build: 1 token, then chunks, then singles
    c2 = new_cache(w, p)
    lens = [0, 0, 0]
    for target in ([1, 1, 1], [130, 64, 700], [131, 200, 2999], list(w.ctx)):
        append(c2, w, lens, target)
        lens = target
    torch.cuda.synchronize()
    assert c1.device_status() == 0 and c2.device_status() == 0
    assert torch.equal(c1.centroids, c2.centroids)  # same bits, whatever the append pattern
    for b in range(3):
        L = w.ctx[b]
        K = workloads.keys(w, b, 0, L)
        assert torch.equal(read_pages(c1, b, L, "k").view(torch.uint8), K.view(torch.uint8))
        assert torch.equal(read_pages(c1, b, L, "v").view(torch.uint8),
                           workloads.values(w, b, 0, L).view(torch.uint8))
        C = oracle.centroids(K, B)
        ids = p.table[b, :C.shape[0]].long()
        got = c1.centroids.cpu()[ids].double().numpy()
        # fp32 relative 1e-6, relative to the block's mean key magnitude (the
        # scale of the rounding error of a sum of fp32 terms)
        Kd = K.double().numpy()
        nb = C.shape[0]
        pad = np.zeros((nb * B - L,) + Kd.shape[1:])
        scale = np.abs(np.concatenate([Kd, pad])).reshape(nb, B, w.hkv, d).sum(1)
        scale /= np.minimum(B, L - np.arange(nb) * B)[:, None, None]
        assert np.all(np.abs(got - C) <= 1e-6 * np.maximum(np.abs(C), scale.mean(-1, keepdims=True)))


# ---------------------------------------------------------------------------
# prefill: selection + attention
# ---------------------------------------------------------------------------
PREFILL_CASES = [
    # (name, overrides)
    ("g8_b128", dict(ctx=(1200,), top_k=4)),
    ("g8_b128_k16", dict(ctx=(2200,), top_k=16)),
    ("g16_b128", dict(ctx=(900,), hq=64, hkv=4, top_k=3)),
    ("g8_b64", dict(ctx=(700,), block=64, top_k=5)),
    ("g4_simt", dict(ctx=(500,), hq=16, hkv=4, top_k=3)),
    # no planted blocks: selections differ from token to token, so tiles walk
    # wide unions and the softmax takes its one-half-of-a-warp path often
    ("g16_b128_unplanted", dict(ctx=(2048,), hq=64, hkv=4, top_k=6, planted=(0, 0))),
    ("g8_b128_unplanted", dict(ctx=(4096,), top_k=8, planted=(0, 0))),
]


def _run_prefill(w, cache, device=DEV):
    T = w.ctx[0]
    append(cache, w, [0], [T])
    q = workloads.queries_prefill(w, 0, 0, T, device)
    cu = msa.cu_seqlens([T], device)
    idx, sc = msa.select_topk(cache, q, w.top_k, cu_q=cu, max_rows_per_seq=T, want_scores=True)
    out, lse = msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=T)
    torch.cuda.synchronize()
    return q, cu, idx, sc, out, lse


@pytest.mark.parametrize("name,over", PREFILL_CASES, ids=[c[0] for c in PREFILL_CASES])
def test_prefill_end_to_end(name, over):
    w = workloads.prefill_bf16(**over)
    p = workloads.paging(w)
    cache = new_cache(w, p)
    q, cu, idx, sc, out, lse = _run_prefill(w, cache)
    assert cache.device_status() == 0
    T = w.ctx[0]
    pos = np.arange(T)
    orc = oracle_rows(w, 0, T, pos, q.cpu())
    stats = check_selection(idx.cpu().numpy(), orc, pos, w.top_k, w.block)
    assert stats["protected_frac"] > 0.3
    # attention checked on the oracle's own indices (removes tie ambiguity)
    oi = torch.from_numpy(orc["idx"]).to(DEV)
    out2, lse2 = msa.sparse_attn_prefill(cache, q, oi, cu_q=cu, max_rows_per_seq=T)
    torch.cuda.synchronize()
    compare(out2, orc["out"], w.dtype)
    assert np.abs(lse2.cpu().double().numpy() - orc["lse"]).max() < 2e-3
    # where the selections agree the end-to-end output matches too
    same = (idx.cpu().numpy() == orc["idx"]).all(-1)             # [T, Hkv]
    rows_ok = same.all(-1)
    assert rows_ok.mean() > 0.5
    compare(out[torch.from_numpy(rows_ok).to(DEV)], orc["out"][rows_ok], w.dtype)


def test_tiny_f32_prefill_and_decode():
    """The tiny fp32 workload: full prefill of 1024 rows, then decode of the last
    query after 1023 cached tokens; decode must equal prefill row 1023."""
    w = workloads.tiny_f32()
    p = workloads.paging(w)
    cache = new_cache(w, p)
    q, cu, idx, sc, out, lse = _run_prefill(w, cache)
    T = w.ctx[0]
    pos = np.arange(T)
    orc = oracle_rows(w, 0, T, pos, q.cpu())
    check_selection(idx.cpu().numpy(), orc, pos, w.top_k, w.block)
    oi = torch.from_numpy(orc["idx"]).to(DEV)
    out2, lse2 = msa.sparse_attn_prefill(cache, q, oi, cu_q=cu, max_rows_per_seq=T)
    torch.cuda.synchronize()
    compare(out2, orc["out"], "f32")
    assert np.abs(lse2.cpu().double().numpy() - orc["lse"]).max() < 1e-5
    # decode: cache of 1023 tokens, append token 1023, attend
    c2 = new_cache(w, p)
    append(c2, w, [0], [T - 1])
    append(c2, w, [T - 1], [T])
    qd = q[T - 1:].contiguous()
    di, _ = msa.select_topk(c2, qd, w.top_k)
    do, dl = msa.sparse_attn_decode(c2, qd, di)
    torch.cuda.synchronize()
    assert torch.equal(di, idx[T - 1:])
    compare(do, orc["out"][T - 1:], "f32")
    assert torch.allclose(do, out[T - 1:], atol=1e-6, rtol=0)


def test_prefill_page_permutation_invariance():
    w = workloads.prefill_bf16(ctx=(1100,), top_k=5)
    p1 = workloads.paging(w)
    p2 = workloads.paging(w, spare_pages=7)   # different pool size -> different permutation
    assert not torch.equal(p1.table, p2.table[:, :p1.table.shape[1]])
    r1 = _run_prefill(w, new_cache(w, p1))
    r2 = _run_prefill(w, new_cache(w, p2))
    assert torch.equal(r1[2], r2[2])
    assert torch.equal(r1[4].view(torch.int16), r2[4].view(torch.int16))


def test_chunked_prefill_matches_full():
    """Rows appended in two chunks (q_pos0 > 0 through cu_q + seq_lens) equal the
    same rows of a one-shot prefill."""
    w = workloads.prefill_bf16(ctx=(1500,), top_k=6)
    p = workloads.paging(w)
    full = _run_prefill(w, new_cache(w, p))
    cache = new_cache(w, p)
    T, T0 = 1500, 1000
    append(cache, w, [0], [T0])
    append(cache, w, [T0], [T])
    q = workloads.queries_prefill(w, 0, T0, T, DEV)
    cu = msa.cu_seqlens([T - T0], DEV)
    idx, _ = msa.select_topk(cache, q, w.top_k, cu_q=cu, max_rows_per_seq=T - T0)
    out, _ = msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=T - T0)
    torch.cuda.synchronize()
    assert torch.equal(idx, full[2][T0:])
    compare(out, full[4][T0:].float().cpu().double().numpy(), "bf16")
    # and the chunk's selection against the oracle at positions T0 .. T-1
    pos = np.arange(T0, T)
    orc = oracle_rows(w, 0, T, pos, q.cpu())
    check_selection(idx.cpu().numpy(), orc, pos, w.top_k, w.block)
    same = (idx.cpu().numpy() == orc["idx"]).all(-1).all(-1)
    compare(out[torch.from_numpy(same).to(DEV)], orc["out"][same], "bf16")


def test_prefill_batch_varlen_chunked_and_index_edges():
    """Three sequences in one call: a full prefill of 700 rows, a chunk of 900
    rows after 1000 cached tokens, and 2600 rows (ragged last query tiles); then
    the same call with a repeated block in some rows (counted once) and rows
    without any block (A = 0, lse = -inf)."""
    w = workloads.prefill_bf16(batch=3, ctx=(700, 1900, 2600), top_k=8)
    p = workloads.paging(w)
    cache = new_cache(w, p)
    first = [0, 1000, 0]
    append(cache, w, [0, 0, 0], first)
    append(cache, w, first, list(w.ctx))
    n = [w.ctx[b] - first[b] for b in range(3)]
    q = torch.cat([workloads.queries_prefill(w, b, first[b], w.ctx[b], DEV) for b in range(3)])
    cu = msa.cu_seqlens(n, DEV)
    idx, _ = msa.select_topk(cache, q, w.top_k, cu_q=cu, max_rows_per_seq=max(n))
    out, lse = msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=max(n))
    # edge rows: slot 1 repeats slot 0 (the block counts once), or no block at all
    rng = np.random.default_rng(7)
    idx_e = idx.cpu().numpy().copy()
    rows = rng.choice(len(idx_e), 300, replace=False)
    dup, empty = rows[:200], rows[200:]
    for r in dup:
        g = int(rng.integers(w.hkv))
        if idx_e[r, g, 1] >= 0:
            idx_e[r, g, 1] = idx_e[r, g, 0]
    idx_e[empty] = -1
    ref_e = idx_e
    out_e, lse_e = msa.sparse_attn_prefill(cache, q, torch.from_numpy(idx_e).to(DEV), cu_q=cu,
                                           max_rows_per_seq=max(n))
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    gi = idx.cpu().numpy()
    r0 = 0
    for b in range(3):
        pos = np.arange(first[b], w.ctx[b])
        sl = slice(r0, r0 + n[b])
        qb = q[sl].cpu()
        # selection of every row (the chunk's rows sit after cached tokens)
        # against the oracle's own top-k at those positions
        sel = check_selection(gi[sl], oracle_rows(w, b, w.ctx[b], pos, qb), pos, w.top_k,
                              w.block)
        assert sel["protected_frac"] > 0.3
        orc = oracle_rows(w, b, w.ctx[b], pos, qb, idx=gi[sl])
        compare(out[sl], orc["out"], w.dtype)
        assert np.abs(lse[sl].cpu().double().numpy() - orc["lse"]).max() < 2e-3
        orc_e = oracle_rows(w, b, w.ctx[b], pos, qb, idx=ref_e[sl])
        keep = ~np.isin(np.arange(r0, r0 + n[b]), empty)
        compare(out_e[sl][torch.from_numpy(keep).to(DEV)], orc_e["out"][keep], w.dtype)
        le = lse_e[sl].cpu().double().numpy()
        assert np.abs(le[keep] - orc_e["lse"][keep]).max() < 2e-3
        r0 += n[b]
    assert torch.all(out_e[torch.from_numpy(empty).to(DEV)] == 0)
    assert torch.all(torch.isneginf(lse_e[torch.from_numpy(empty).to(DEV)]))


EMPTY_CASES = [("g8_b128", dict(ctx=(700,), top_k=4)),
               ("g16_b128", dict(ctx=(600,), hq=64, hkv=4, top_k=3)),
               ("g8_b64", dict(ctx=(500,), block=64, top_k=5)),
               ("g4_simt", dict(ctx=(400,), hq=16, hkv=4, top_k=3))]


@pytest.mark.parametrize("name,over", EMPTY_CASES, ids=[c[0] for c in EMPTY_CASES])
def test_rows_without_blocks(name, over):
    """A row whose block list is all -1 attends to nothing: A = 0, lse = -inf,
    on every prefill path; the other rows are unaffected."""
    w = workloads.prefill_bf16(**over)
    cache = new_cache(w, workloads.paging(w))
    T = w.ctx[0]
    append(cache, w, [0], [T])
    q = workloads.queries_prefill(w, 0, 0, T, DEV)
    cu = msa.cu_seqlens([T], DEV)
    idx, _ = msa.select_topk(cache, q, w.top_k, cu_q=cu, max_rows_per_seq=T)
    ref, ref_lse = msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=T)
    empty = torch.arange(3, T, 7, device=DEV)
    idx2 = idx.clone()
    idx2[empty] = -1
    out, lse = msa.sparse_attn_prefill(cache, q, idx2, cu_q=cu, max_rows_per_seq=T)
    # a block repeated in the adjacent slot counts once: same as -1 in that slot
    dup = torch.arange(200, T, 11, device=DEV)
    dup = dup[(idx[dup, :, 1] >= 0).all(-1)]
    idx3, idx4 = idx.clone(), idx.clone()
    idx3[dup, :, 1] = idx3[dup, :, 0]
    idx4[dup, :, 1] = -1
    out3, _ = msa.sparse_attn_prefill(cache, q, idx3, cu_q=cu, max_rows_per_seq=T)
    out4, _ = msa.sparse_attn_prefill(cache, q, idx4, cu_q=cu, max_rows_per_seq=T)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert torch.all(out[empty] == 0) and torch.all(torch.isneginf(lse[empty]))
    keep = torch.ones(T, dtype=torch.bool, device=DEV)
    keep[empty] = False
    assert torch.equal(out[keep].view(torch.int16), ref[keep].view(torch.int16))
    assert len(dup) > 10
    assert (out3[dup].float() - out4[dup].float()).abs().max().item() < 1e-6
    assert not torch.equal(out3[dup], ref[dup])   # the lists did change


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------
DECODE_CASES = [
    ("paged_g4", lambda: workloads.paged_decode_bf16(batch=4, ctx=(3000, 4095, 4096, 5000))),
    ("long_g8_b128", lambda: workloads.decode_1m_bf16(ctx=(40000,), steps=3)),
    ("varlen_g16", lambda: workloads.varlen_decode_bf16(batch=5, len_range=(1000, 20000))),
    # k-1 > 64: the tournament merge; k = 2: one-key chunk lists
    ("topk100", lambda: workloads.paged_decode_bf16(batch=3, ctx=(9000, 12000, 20000), top_k=100)),
    ("topk2", lambda: workloads.paged_decode_bf16(batch=2, ctx=(5000, 700), top_k=2,
                                                  planted=(1, 1))),
]


def test_decode_repeated_and_empty_block_lists():
    """Decode attention: an adjacent repeat of a block counts once, a sequence
    whose list is all -1 gives 0 and lse = -inf."""
    w = workloads.paged_decode_bf16(batch=3, ctx=(3000, 5000, 4096))
    p = workloads.paging(w)
    cache = new_cache(w, p)
    lens = fill_context(cache, w)
    append(cache, w, lens, [L + 1 for L in lens])
    q = workloads.queries_decode(w, 0, DEV)
    idx, _ = msa.select_topk(cache, q, w.top_k)
    ref, _ = msa.sparse_attn_decode(cache, q, idx)
    idx3, idx4 = idx.clone(), idx.clone()
    for s_ in (1, 9, 17):   # repeats inside and across the split boundaries
        idx3[0, :, s_] = idx3[0, :, s_ - 1]
        idx4[0, :, s_] = -1
    idx3[2] = -1
    idx4[2] = -1
    o3, l3 = msa.sparse_attn_decode(cache, q, idx3)
    o4, l4 = msa.sparse_attn_decode(cache, q, idx4)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    assert (o3[0].float() - o4[0].float()).abs().max().item() < 1e-6
    assert not torch.equal(o3[0], ref[0])
    assert torch.equal(o3[1].view(torch.int16), ref[1].view(torch.int16))
    assert torch.all(o3[2] == 0) and torch.all(torch.isneginf(l3[2]))


@pytest.mark.parametrize("name,make", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_end_to_end(name, make):
    w = make()
    p = workloads.paging(w)
    cache = new_cache(w, p)
    lens = fill_context(cache, w)
    hit = [0, 0]   # planted blocks selected / planted blocks
    for step in range(w.steps):
        after = [w.ctx[b] + step + 1 for b in range(w.batch)]
        append(cache, w, lens, after)
        lens = after
        q = workloads.queries_decode(w, step, DEV)
        idx, _ = msa.select_topk(cache, q, w.top_k)
        out, lse = msa.sparse_attn_decode(cache, q, idx)
        torch.cuda.synchronize()
        assert cache.device_status() == 0
        oidx, refs = [], []
        for b in range(w.batch):
            L = lens[b]
            pos = np.array([L - 1])
            K, V = workloads.keys(w, b, 0, L), workloads.values(w, b, 0, L)
            orc = oracle.forward(q[b:b + 1].cpu(), K, V, pos, w.block, w.top_k, w.softmax_scale)
            check_selection(idx[b:b + 1].cpu().numpy(), orc, pos, w.top_k, w.block)
            for g, blocks in enumerate(workloads.planted_blocks(w)[b]):
                hit[0] += len(set(blocks) & set(idx[b, g].tolist()))
                hit[1] += len(blocks)
            if np.array_equal(orc["idx"], idx[b:b + 1].cpu().numpy()):
                compare(out[b:b + 1], orc["out"], w.dtype)
                assert np.abs(lse[b].cpu().double().numpy() - orc["lse"][0]).max() < 2e-3
            oidx.append(orc["idx"])
            refs.append(orc["out"])
        # attention on the oracle's indices, all sequences at once
        o2, _ = msa.sparse_attn_decode(cache, q, torch.from_numpy(np.concatenate(oidx)).to(DEV))
        torch.cuda.synchronize()
        compare(o2, np.concatenate(refs), w.dtype)
    # the planted "needle" blocks are found far more often than chance
    assert hit[1] == 0 or hit[0] >= 0.75 * hit[1], hit


def test_decode_equals_prefill_rows():
    """Selecting and attending the last rows one at a time through the decode
    entry points gives the prefill selection and (within bf16 tolerance) output."""
    w = workloads.prefill_bf16(ctx=(1300,), top_k=5, hq=16, hkv=2)
    p = workloads.paging(w)
    full = _run_prefill(w, new_cache(w, p))
    cache = new_cache(w, p)
    T = 1300
    append(cache, w, [0], [T - 3])
    for t in range(T - 3, T):
        append(cache, w, [t], [t + 1])
        q = full[0][t:t + 1].contiguous()
        di, _ = msa.select_topk(cache, q, w.top_k)
        do, _ = msa.sparse_attn_decode(cache, q, di)
        torch.cuda.synchronize()
        assert torch.equal(di, full[2][t:t + 1])
        compare(do, full[4][t:t + 1].float().cpu().double().numpy(), "bf16")


# ---------------------------------------------------------------------------
# error paths (no fault, no trap: host status codes and the device status word)
# ---------------------------------------------------------------------------
def test_host_argument_errors():
    w = workloads.prefill_bf16(ctx=(256,), top_k=2)
    p = workloads.paging(w)
    cache = new_cache(w, p)
    append(cache, w, [0], [256])
    q = workloads.queries_prefill(w, 0, 0, 256, DEV)
    cu = msa.cu_seqlens([256], DEV)
    with pytest.raises(msa.MsaError) as e:
        msa.select_topk(cache, q, 0, cu_q=cu, max_rows_per_seq=256)
    assert e.value.status == msa.MSA_ERR_UNSUPPORTED
    with pytest.raises(msa.MsaError) as e:
        msa.select_topk(cache, q, 300, cu_q=cu, max_rows_per_seq=256)
    assert e.value.status == msa.MSA_ERR_UNSUPPORTED
    idx, _ = msa.select_topk(cache, q, 2, cu_q=cu, max_rows_per_seq=256)
    small = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(msa.MsaError) as e:
        msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=256, workspace=small)
    assert e.value.status == msa.MSA_ERR_WORKSPACE
    bad = msa.PagedKVCache(cache.k_pages, cache.v_pages, cache.centroids, cache.page_table,
                           cache.seq_lens, cache.status_word, num_q_heads=33)
    with pytest.raises(msa.MsaError) as e:
        msa.select_topk(bad, q, 2, cu_q=cu, max_rows_per_seq=256)
    assert e.value.status == msa.MSA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert cache.device_status() == 0


def test_device_status_on_bad_page_and_length():
    w = workloads.paged_decode_bf16(batch=2, ctx=(500, 700))
    p = workloads.paging(w)
    cache = new_cache(w, p)
    fill_context(cache, w)
    append(cache, w, list(w.ctx), [w.ctx[0] + 1, w.ctx[1] + 1])
    q = workloads.queries_decode(w, 0, DEV)
    cache.page_table[1, 3] = p.num_pages + 5          # corrupt one page id (host-side injection)
    idx, _ = msa.select_topk(cache, q, w.top_k)
    msa.sparse_attn_decode(cache, q, idx)
    torch.cuda.synchronize()
    assert cache.device_status() & msa.MSA_DEV_BAD_PAGE
    cache.clear_status()
    cache.page_table.copy_(p.table.to(DEV))
    cache.seq_lens[0] = p.max_blocks * w.block + 1    # beyond capacity
    idx, _ = msa.select_topk(cache, q, w.top_k)
    torch.cuda.synchronize()
    assert cache.device_status() & msa.MSA_DEV_BAD_LENGTH
    # the context still works afterwards
    cache.clear_status()
    cache.seq_lens.copy_(torch.tensor([w.ctx[0] + 1, w.ctx[1] + 1], dtype=torch.int32))
    idx, _ = msa.select_topk(cache, q, w.top_k)
    msa.sparse_attn_decode(cache, q, idx)
    torch.cuda.synchronize()
    assert cache.device_status() == 0


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.mark.parametrize("name,make", [
    ("paged_g4", lambda: workloads.paged_decode_bf16(batch=4, ctx=(3000, 4095, 4096, 5000))),
    ("long_g8_b128", lambda: workloads.decode_1m_bf16(ctx=(40000,), steps=1)),
], ids=["paged_g4", "long_g8_b128"])
def test_decode_graph_replays_and_shared_workspace(name, make):
    """The decode attention publishes the parts of split (sequence, group) units
    under a tag drawn per host call, which a CUDA graph captures once, and the
    finishing CTA clears the flags it read. Replays of one graph, and two graphs
    (two tags) alternating on one workspace, must give the eager call's bits."""
    w = make()
    p = workloads.paging(w)
    cache = new_cache(w, p)
    lens = fill_context(cache, w)
    after = [L + 1 for L in lens]
    append(cache, w, lens, after)
    q0 = workloads.queries_decode(w, 0, DEV)
    q1 = (q0.float() * 0.5).to(q0.dtype)
    ws = torch.empty(msa.workspace_size(msa.MSA_OP_DECODE, cache, w.batch, 1, w.top_k),
                     dtype=torch.uint8, device=DEV)
    idx0, _ = msa.select_topk(cache, q0, w.top_k)
    idx1, _ = msa.select_topk(cache, q1, w.top_k)
    ref0, lse0 = msa.sparse_attn_decode(cache, q0, idx0, workspace=ws)
    ref1, lse1 = msa.sparse_attn_decode(cache, q1, idx1, workspace=ws)
    torch.cuda.synchronize()
    out0, l0 = torch.empty_like(ref0), torch.empty_like(lse0)
    out1, l1 = torch.empty_like(ref1), torch.empty_like(lse1)
    graphs = []
    for q, idx, o, l in ((q0, idx0, out0, l0), (q1, idx1, out1, l1)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            msa.sparse_attn_decode(cache, q, idx, out=o, lse=l, workspace=ws)
        graphs.append(g)
    torch.cuda.synchronize()
    for rep in range(3):
        for g, o, l, ro, rl in ((graphs[0], out0, l0, ref0, lse0), (graphs[1], out1, l1, ref1, lse1)):
            o.fill_(float("nan"))
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(_bits(o), _bits(ro)), (name, rep)
            assert torch.equal(_bits(l), _bits(rl)), (name, rep)
    for rep in range(2):  # one graph replayed back to back
        graphs[0].replay()
    torch.cuda.synchronize()
    assert torch.equal(_bits(out0), _bits(ref0))
    assert cache.device_status() == 0


@pytest.mark.parametrize("which", [0, 1], ids=["mbarrier_phase", "published_flag"])
def test_bounded_wait_gives_up_and_context_survives(which):
    """A device wait on something never completed (an mbarrier phase nothing
    arrives at, a flag nothing publishes) gives up after about a second with
    MSA_DEV_TIMEOUT, and the context keeps working: a decode step afterwards
    matches the oracle."""
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    msa.selftest_bounded_wait(which, st)
    b.record()
    torch.cuda.synchronize()
    assert st.item() == msa.MSA_DEV_TIMEOUT
    assert 900.0 <= a.elapsed_time(b) <= 5000.0
    w = workloads.paged_decode_bf16(batch=2, ctx=(500, 700))
    p = workloads.paging(w)
    cache = new_cache(w, p)
    lens = fill_context(cache, w)
    after = [L + 1 for L in lens]
    append(cache, w, lens, after)
    q = workloads.queries_decode(w, 0, DEV)
    idx, _ = msa.select_topk(cache, q, w.top_k)
    out, _ = msa.sparse_attn_decode(cache, q, idx)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    for bq in range(w.batch):
        L = after[bq]
        K, V = workloads.keys(w, bq, 0, L), workloads.values(w, bq, 0, L)
        O, _ = oracle.attend(q[bq:bq + 1].cpu(), K, V, np.array([L - 1]),
                             idx[bq:bq + 1].cpu().numpy(), w.block, w.softmax_scale)
        compare(out[bq:bq + 1], O, "bf16")
