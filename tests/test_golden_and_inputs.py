"""Oracle regression record and input-generator determinism (CPU only)."""
import json
import os

import numpy as np
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_f32_rows.json")


def test_oracle_matches_regression_record():
    rec = json.load(open(GOLDEN))
    w = workloads.tiny_f32()
    L = w.ctx[0]
    K, V = workloads.keys(w, 0, 0, L), workloads.values(w, 0, 0, L)
    Q = workloads.queries_prefill(w, 0, 0, L)
    rows = rec["rows"]
    r = oracle.forward(Q[rows], K, V, np.array(rows), w.block, w.top_k, w.softmax_scale)
    assert r["idx"][:, 0].tolist() == rec["idx"]
    assert np.max(np.abs(r["lse"] - np.array(rec["lse"]))) < 1e-12
    assert np.max(np.abs(r["out"][-1] - np.array(rec["out_row_1023"]))) < 1e-12
    assert np.max(np.abs(r["centroids"][3, 0] - np.array(rec["centroid_block_3"]))) < 1e-12


def test_generator_slices_are_consistent():
    w = workloads.prefill_bf16(ctx=(1024,))
    a = workloads.keys(w, 0, 0, 300)
    b = workloads.keys(w, 0, 100, 300)
    assert torch.equal(a[100:].view(torch.int16), b.view(torch.int16))
    q1 = workloads.queries_prefill(w, 0, 0, 64)
    q2 = workloads.queries_prefill(w, 0, 32, 64)
    assert torch.equal(q1[32:].view(torch.int16), q2.view(torch.int16))


def test_generator_moments_and_planting():
    z = workloads.gauss((1, 2, 3), 0, 1 << 20, "cpu").to(torch.float64)
    assert abs(float(z.mean())) < 5e-3 and abs(float(z.std()) - 1.0) < 5e-3
    w = workloads.prefill_bf16(ctx=(4096,))
    planted = workloads.planted_blocks(w)[0]
    assert all(len(p) == 8 for p in planted)
    K = workloads.keys(w, 0, 0, 4096).to(torch.float64)
    u = workloads._directions(w)[0].to(torch.float64)
    for g in range(w.hkv):
        proj = (K[:, g] @ u[g]).view(-1, w.block).mean(1)
        for j in range(4096 // w.block):
            if j in planted[g]:
                assert proj[j] > 1.0
            else:
                assert abs(float(proj[j])) < 0.5


def test_paging_is_a_permutation():
    w = workloads.paged_decode_bf16(batch=3, ctx=(1000, 64, 129))
    p = workloads.paging(w)
    used = p.table[p.table >= 0]
    assert sorted(used.tolist()) == list(range(p.num_pages))
    assert p.max_blocks == -(-1001 // 64)
