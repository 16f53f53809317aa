"""The algorithmic work the bench divides by (the roofline numerators), on the
CPU: the attended (query, key) pair count of a causal block-sparse prefill
against an explicit mask, and the decode byte accounting against a small case
worked by hand and against its split into the two calls."""
import dataclasses

import numpy as np
import pytest

import bench
import workloads


def _pairs_brute_force(T, B, k):
    """Row t attends to its own block's keys up to t and to k-1 complete past
    blocks (all of them when fewer): count the (t, u) pairs of that mask."""
    n = 0
    for t in range(T):
        own = t // B
        past = min(k - 1, own)
        for u in range(t + 1):
            j = u // B
            if j == own or j >= own - past:  # any k-1 past blocks give the same count
                n += 1
    return n


@pytest.mark.parametrize("T,B,k", [(1, 64, 4), (64, 64, 1), (700, 64, 5), (1000, 128, 3),
                                   (4096, 64, 16)])
def test_attended_pairs_matches_the_mask(T, B, k):
    assert bench.attended_pairs(T, B, k) == _pairs_brute_force(T, B, k)


def test_decode_bytes_by_hand():
    """One sequence of 300 cached tokens + 1 new, block 64, top-k 4, 1 KV head
    of 2 query heads, d 8: own block 4 (positions 256..300, 45 keys), 4 complete
    past blocks of which 3 are kept."""
    w = dataclasses.replace(workloads.paged_decode_bf16(), batch=1, ctx=(300,), block=64,
                            top_k=4, hkv=1, hq=2, d=8)
    centroids = 4 * 8 * 4                 # every complete past block's centroid row, fp32
    kv = (3 * 64 + 45) * 8 * 2 * 2        # K and V rows of the kept blocks + own block, bf16
    q_out = 2 * 2 * 8 * 2                 # q in and out, bf16
    append = 2 * 1 * 8 * 2 + 1 * 8 * 4    # the new K/V row and its block's centroid
    assert bench.decode_bytes(w) == centroids + kv + q_out + append
    sel, att = bench.decode_call_bytes(w)
    assert sel == centroids + 2 * 8 * 2
    assert att == kv + q_out


@pytest.mark.parametrize("make", [workloads.paged_decode_bf16, workloads.varlen_decode_bf16,
                                  workloads.decode_1m_bf16])
def test_decode_bytes_equal_the_calls_plus_the_append(make):
    w = make()
    sel, att = bench.decode_call_bytes(w)
    append = w.batch * (2 * w.hkv * w.d * 2 + w.hkv * w.d * 4)
    q_in_counted_twice = w.batch * w.hq * w.d * 2  # each call reads q
    assert bench.decode_bytes(w) == sel + att + append - q_in_counted_twice


def test_prefill_headline_numerator():
    """The prefill roofline's algorithmic flops per launch: 4 * d flops per
    attended (query head, key) pair, 32 query heads, T = 32768, block 128,
    top-k 16 (the figure the bench line reports)."""
    w = workloads.prefill_bf16()
    flops = 4 * w.d * w.hq * bench.attended_pairs(w.ctx[0], w.block, w.top_k)
    assert flops == 1033208070144
