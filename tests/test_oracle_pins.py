"""Pins for the CPU oracle: each check ties it to something other than itself.

* library routines: torch's scaled_dot_product_attention and logsumexp (CPU,
  float64) for the cases where the method reduces to dense or block-local
  causal attention;
* closed forms: centroids of a ramp of keys, scores of one-hot queries, the
  selection and gap of monotone score ramps;
* brute force: enumeration of every candidate subset on tiny inputs;
* invariants: softmax weights are non-negative, sum to one and vanish off the
  attended set; one-key rows return that key's value exactly.

The method: "MiniMax Sparse Attention" (staik.se), method paragraph (per-GQA-
group top-k over KV blocks, then exact attention over them); "Art of Focus:
Ling 2.0 ...", "Summarizing the Breakthrough" (block representations in a
cache, GQA-shared selection); "Sparse Attention + Linear Backbones", section
5.5 (softmax(q k^T / sqrt(d)) v over the selected set).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import workloads


def _rand(shape, seed, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64).to(dtype)


def _sdpa_ref(Q, K, V, mask, scale):
    """torch SDPA in float64 with K/V heads repeated for GQA. mask: [R, L] bool."""
    G = Q.shape[1] // K.shape[1]
    q = Q.to(torch.float64).permute(1, 0, 2)                       # [Hq, R, d]
    k = K.to(torch.float64).repeat_interleave(G, dim=1).permute(1, 0, 2)
    v = V.to(torch.float64).repeat_interleave(G, dim=1).permute(1, 0, 2)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("L,B,d,hq,hkv", [(200, 16, 32, 6, 2), (97, 8, 16, 4, 4), (64, 64, 64, 4, 1)])
def test_dense_pin(dtype, L, B, d, hq, hkv):
    """k >= number of blocks: the method is dense causal attention."""
    Q, K, V = _rand((L, hq, d), 1, dtype), _rand((L, hkv, d), 2, dtype), _rand((L, hkv, d), 3, dtype)
    nblk = -(-L // B)
    pos = np.arange(L)
    scale = 1.0 / math.sqrt(d)
    r = oracle.forward(Q, K, V, pos, B, nblk + 1, scale)
    causal = torch.ones(L, L, dtype=torch.bool).tril()
    ref = _sdpa_ref(Q, K, V, causal, scale)
    assert np.max(np.abs(r["out"] - ref)) < 1e-12
    # lse against the library logsumexp of the masked logits
    G = hq // hkv
    logits = torch.einsum("rhd,uhd->hru", Q.to(torch.float64),
                          K.to(torch.float64).repeat_interleave(G, dim=1)) * scale
    logits = logits.masked_fill(~causal, float("-inf"))
    lse_ref = torch.logsumexp(logits, dim=-1).T.numpy()
    assert np.max(np.abs(r["lse"] - lse_ref)) < 1e-10


@pytest.mark.parametrize("L,B", [(130, 16), (64, 8)])
def test_block_local_pin(L, B):
    """k = 1: each query attends causally inside its own block only."""
    d, hq, hkv = 24, 4, 2
    Q, K, V = _rand((L, hq, d), 4), _rand((L, hkv, d), 5), _rand((L, hkv, d), 6)
    pos = np.arange(L)
    scale = 1.0 / math.sqrt(d)
    r = oracle.forward(Q, K, V, pos, B, 1, scale)
    t = torch.arange(L)
    mask = (t[None, :] <= t[:, None]) & ((t[None, :] // B) == (t[:, None] // B))
    ref = _sdpa_ref(Q, K, V, mask, scale)
    assert np.max(np.abs(r["out"] - ref)) < 1e-12
    # rows that open a block see exactly one key: output is that value, exactly
    for t0 in range(0, L, B):
        for h in range(hq):
            assert np.array_equal(r["out"][t0, h], V[t0, h // (hq // hkv)].to(torch.float64).numpy())


def test_softmax_weights():
    """One-hot values expose the weights: >= 0, sum to 1, zero off the attended set."""
    L, B, d, hq, hkv, k = 40, 5, 64, 2, 1, 3
    Q, K = _rand((L, hq, d), 7) * 2.0, _rand((L, hkv, d), 8)
    V = torch.zeros(L, hkv, d)
    for u in range(L):
        V[u, 0, u] = 1.0
    pos = np.arange(L)
    r = oracle.forward(Q, K, V, pos, B, k, 0.125)
    W = r["out"][:, :, :L]
    assert np.all(W >= 0)
    assert np.max(np.abs(W.sum(-1) - 1.0)) < 1e-12
    for t in range(L):
        allowed = set()
        for j in r["idx"][t, 0]:
            if j >= 0:
                allowed |= {u for u in range(j * B, (j + 1) * B) if u <= t}
        off = [u for u in range(L) if u not in allowed]
        assert np.all(W[t, :, off] == 0.0)


def test_centroid_closed_form():
    """Keys k[u] = u * e1 give c_j = (jB + (n_j - 1)/2) e1, n_j tokens present."""
    L, B, d = 203, 16, 8
    K = torch.zeros(L, 2, d)
    K[:, :, 0] = torch.arange(L, dtype=torch.float32)[:, None]
    C = oracle.centroids(K, B)
    assert C.shape == (13, 2, d)
    for j in range(13):
        n = min(B, L - j * B)
        assert C[j, 0, 0] == j * B + (n - 1) / 2.0
        assert C[j, 1, 0] == j * B + (n - 1) / 2.0
        assert np.all(C[j, :, 1:] == 0.0)


def test_scores_one_hot_queries():
    """One-hot queries pick centroid coordinates: s_j = sum_h c_j[i_h]; NaN if j >= b(t)."""
    L, B, d, hq, hkv = 64, 8, 6, 4, 2
    K = _rand((L, hkv, d), 9)
    C = oracle.centroids(K, B)
    Q = torch.zeros(3, hq, d)
    hot = [[0, 5, 2, 2], [1, 1, 4, 3], [3, 0, 0, 5]]
    for r in range(3):
        for h in range(hq):
            Q[r, h, hot[r][h]] = 1.0
    pos = np.array([63, 40, 17])
    S = oracle.scores(Q, pos, C, B)
    for r in range(3):
        bt = pos[r] // B
        for g in range(hkv):
            for j in range(C.shape[0]):
                if j >= bt:
                    assert np.isnan(S[r, g, j])
                else:
                    want = C[j, g, hot[r][2 * g]] + C[j, g, hot[r][2 * g + 1]]
                    assert abs(S[r, g, j] - want) < 1e-15


def _brute_force(scores_row, bt, k):
    """Best (k-1)-subset of past blocks under (score desc, index asc) - by enumeration."""
    take = min(k - 1, bt)
    best = None
    for comb in itertools.combinations(range(bt), take):
        keylist = sorted(((scores_row[j], -j) for j in comb), reverse=True)
        if best is None or keylist > best[0]:
            best = (keylist, comb)
    chosen = sorted(set(best[1]) | {bt})
    rejected = [scores_row[j] for j in range(bt) if j not in best[1]]
    gap = (min(scores_row[j] for j in best[1]) - max(rejected)) if (take > 0 and rejected) else math.inf
    return chosen, gap


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_selection_brute_force(k):
    L, B, d, hq, hkv = 44, 4, 8, 4, 2
    Q, K = _rand((L, hq, d), 10 + k), _rand((L, hkv, d), 20 + k)
    pos = np.arange(L)
    C = oracle.centroids(K, B)
    S = oracle.scores(Q, pos, C, B)
    idx, gap = oracle.select(S, pos, B, k)
    for t in range(L):
        for g in range(hkv):
            chosen, bgap = _brute_force(S[t, g], t // B, k)
            got = [int(j) for j in idx[t, g] if j >= 0]
            assert got == chosen
            assert list(idx[t, g][len(got):]) == [-1] * (k - len(got))
            if math.isinf(bgap):
                assert math.isinf(gap[t, g])
            else:
                assert abs(gap[t, g] - bgap) < 1e-14


def test_exact_ties_go_to_lower_index():
    """Duplicated blocks score bit-identically; the lower index wins the last slot."""
    L, B, d, hq, hkv, k = 64, 8, 4, 2, 1, 3
    K = torch.zeros(L, hkv, d)
    K[:, 0, 0] = -1.0
    for j in (2, 5):            # two identical high-scoring blocks
        K[j * B:(j + 1) * B, 0, 0] = 3.0
    K[1 * B:2 * B, 0, 0] = 5.0  # one clear winner
    Q = torch.zeros(1, hq, d)
    Q[0, :, 0] = 1.0
    pos = np.array([L - 1])
    C = oracle.centroids(K, B)
    S = oracle.scores(Q, pos, C, B)
    assert S[0, 0, 2] == S[0, 0, 5]
    idx, gap = oracle.select(S, pos, B, k)
    assert list(idx[0, 0]) == [1, 2, 7]
    assert gap[0, 0] == 0.0


def test_all_equal_scores_pick_lowest():
    L, B, d, k = 80, 8, 4, 4
    K = torch.zeros(L, 1, d)
    Q = torch.ones(5, 2, d)
    pos = np.array([79, 70, 31, 24, 8])
    S = oracle.scores(Q, pos, oracle.centroids(K, B), B)
    idx, _ = oracle.select(S, pos, B, k)
    assert list(idx[0, 0]) == [0, 1, 2, 9]
    assert list(idx[1, 0]) == [0, 1, 2, 8]
    assert list(idx[2, 0]) == [0, 1, 2, 3]   # b = 3 = k-1: every past block kept
    assert list(idx[3, 0]) == [0, 1, 2, 3]
    assert list(idx[4, 0]) == [0, 1, -1, -1]


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_score_ramp_closed_form(sign):
    """Block-constant keys sign*j*e1 and queries e1: scores sign*G*j. An increasing
    ramp keeps the k-1 latest past blocks (never a future one), a decreasing ramp
    the k-1 earliest; the gap is G either way."""
    L, B, d, hq, hkv, k = 160, 8, 4, 6, 2, 5
    G = hq // hkv
    K = torch.zeros(L, hkv, d)
    K[:, :, 0] = sign * (torch.arange(L) // B).to(torch.float32)[:, None]
    Q = torch.zeros(L, hq, d)
    Q[:, :, 0] = 1.0
    pos = np.arange(L)
    S = oracle.scores(Q, pos, oracle.centroids(K, B), B)
    idx, gap = oracle.select(S, pos, B, k)
    for t in range(L):
        b = t // B
        for g in range(hkv):
            if b < k:
                want = list(range(b + 1)) + [-1] * (k - b - 1)
            elif sign > 0:
                want = list(range(b - k + 1, b + 1))
            else:
                want = list(range(k - 1)) + [b]
            assert list(idx[t, g]) == want
            if b >= k:
                assert gap[t, g] == G
            else:
                assert math.isinf(gap[t, g])


def test_permuted_index_order_and_row_subsets():
    """Attention does not depend on the order of the index list, and a row
    computed alone equals the same row computed with all others."""
    L, B, d, hq, hkv, k = 96, 8, 16, 4, 2, 4
    Q, K, V = _rand((L, hq, d), 30), _rand((L, hkv, d), 31), _rand((L, hkv, d), 32)
    pos = np.arange(L)
    r = oracle.forward(Q, K, V, pos, B, k, 0.25)
    perm_idx = r["idx"][:, :, ::-1].copy()
    O2, lse2 = oracle.attend(Q, K, V, pos, perm_idx, B, 0.25)
    assert np.max(np.abs(O2 - r["out"])) < 1e-13
    one = oracle.forward(Q[L - 1:], K, V, pos[L - 1:], B, k, 0.25)
    assert np.array_equal(one["idx"][0], r["idx"][L - 1])
    assert np.max(np.abs(one["out"][0] - r["out"][L - 1])) < 1e-15


def test_repeated_and_empty_block_lists():
    """The attended tokens are a set: a block listed twice equals the block
    listed once; a row without any block attends to nothing (O = 0, lse = -inf),
    and its neighbours are unaffected."""
    L, B, d, hq, hkv, k = 64, 8, 16, 4, 2, 4
    Q, K, V = _rand((L, hq, d), 40), _rand((L, hkv, d), 41), _rand((L, hkv, d), 42)
    pos = np.arange(L)
    r = oracle.forward(Q, K, V, pos, B, k, 0.25)
    idx = r["idx"].copy()
    rows = [t for t in range(L) if idx[t, 0, 1] >= 0][:5]
    dup, ref = idx.copy(), idx.copy()
    for t in rows:
        dup[t, 0, 1] = dup[t, 0, 0]
        ref[t, 0, 1] = -1
    Od, ld = oracle.attend(Q, K, V, pos, dup, B, 0.25)
    Or, lr = oracle.attend(Q, K, V, pos, ref, B, 0.25)
    assert np.array_equal(Od, Or) and np.array_equal(ld, lr)
    assert not np.allclose(Od[rows[0]], r["out"][rows[0]])   # the list did change
    empty = idx.copy()
    empty[7] = -1
    Oe, le = oracle.attend(Q, K, V, pos, empty, B, 0.25)
    assert np.all(Oe[7] == 0.0) and np.all(np.isneginf(le[7]))
    others = np.arange(L) != 7
    assert np.array_equal(Oe[others], r["out"][others])


def test_tiny_workload_finds_planted_blocks():
    """Generator + oracle: the tiny workload plants two blocks along the last
    query's mean head direction, so that query ranks them first."""
    w = workloads.tiny_f32()
    L = w.ctx[0]
    K = workloads.keys(w, 0, 0, L)
    V = workloads.values(w, 0, 0, L)
    Q = workloads.queries_prefill(w, 0, 0, L)
    planted = workloads.planted_blocks(w)[0][0]
    assert len(planted) == 2 and all(j < 15 for j in planted)
    r = oracle.forward(Q[L - 1:], K, V, np.array([L - 1]), w.block, w.top_k, w.softmax_scale)
    S = r["scores"][0, 0, :L // w.block - 1]
    assert sorted(np.argsort(-S)[:2].tolist()) == planted
    assert set(planted) <= set(int(j) for j in r["idx"][0, 0])


# ---------------------------------------------------------------------------
# output gate: O = g * A + (1 - g) * X
# ---------------------------------------------------------------------------
def test_gate_special_cases_and_broadcast():
    rng = np.random.default_rng(5)
    A = rng.standard_normal((3, 4, 8))
    X = rng.standard_normal((3, 4, 8))
    one, zero = np.ones((3, 4)), np.zeros((3, 4))
    assert np.array_equal(oracle.gate(A, one, X), A)        # g = 1: attention only
    assert np.array_equal(oracle.gate(A, zero, X), X)       # g = 0: the other branch only
    half = oracle.gate(A, np.full((3, 4), 0.5), X)
    assert np.allclose(half, (A + X) / 2, rtol=0, atol=1e-15)
    # a per-head gate equals the same value repeated over the coordinates
    g = rng.uniform(0, 1, (3, 4))
    assert np.allclose(oracle.gate(A, g, X), oracle.gate(A, np.repeat(g[..., None], 8, -1), X),
                       rtol=0, atol=1e-15)
    # per-coordinate gate: coordinate c of head h uses g[.., h, c] (catches a transposed gate)
    gd = rng.uniform(0, 1, (3, 4, 8))
    r, h, c = 2, 1, 5
    assert oracle.gate(A, gd, X)[r, h, c] == gd[r, h, c] * A[r, h, c] + (1 - gd[r, h, c]) * X[r, h, c]


def test_gate_widens_bf16_branch():
    x = torch.tensor([[[1.5, -2.25]]], dtype=torch.bfloat16)
    A = np.array([[[0.5, 0.25]]])
    out = oracle.gate(A, np.array([[0.25]]), x)
    assert np.array_equal(out, 0.25 * A + 0.75 * np.array([[[1.5, -2.25]]]))


# --------------------------------------------------------------------------
# token-granular variant (indexer over every position, top-K tokens)
# --------------------------------------------------------------------------
def test_token_topk_all_positions_is_dense_causal():
    """K >= L keeps every earlier position: dense causal attention (torch SDPA)."""
    L, d, hq, hkv, hi, di = 70, 16, 4, 2, 3, 8
    Q, K, V = _rand((L, hq, d), 50), _rand((L, hkv, d), 51), _rand((L, hkv, d), 52)
    QI, KI = _rand((L, hi, di), 53), _rand((L, di), 54)
    pos = np.arange(L)
    S = oracle.token_scores(QI, KI, pos)
    idx, gap = oracle.token_select(S, pos, L + 5)
    for r in range(L):
        assert list(idx[r, :r + 1]) == list(range(r + 1)) and np.all(idx[r, r + 1:] == -1)
    assert np.all(np.isinf(gap))
    O, _ = oracle.attend_tokens(Q, K, V, pos, idx, 0.3)
    mask = torch.from_numpy(np.tril(np.ones((L, L), dtype=bool)))
    assert np.max(np.abs(O - _sdpa_ref(Q, K, V, mask, 0.3))) < 1e-12


def test_token_topk_one_is_the_own_position():
    """K = 1 keeps only the query's own position: O = v_t, lse = scale q.k_t."""
    L, d, hq, hkv = 40, 8, 4, 2
    Q, K, V = _rand((L, hq, d), 60), _rand((L, hkv, d), 61), _rand((L, hkv, d), 62)
    pos = np.arange(L)
    S = oracle.token_scores(_rand((L, 2, 8), 63), _rand((L, 8), 64), pos)
    idx, _ = oracle.token_select(S, pos, 1)
    assert np.array_equal(idx[:, 0], pos)
    O, lse = oracle.attend_tokens(Q, K, V, pos, idx, 0.5)
    v, q, k = V.double().numpy(), Q.double().numpy(), K.double().numpy()
    for h in range(hq):
        assert np.array_equal(O[:, h], v[:, h // 2])
        assert np.max(np.abs(lse[:, h] - 0.5 * np.einsum("rd,rd->r", q[:, h], k[:, h // 2]))) < 1e-12


def test_token_select_brute_force_and_ties():
    """Every kept earlier position scores at least as high as every dropped one;
    among equal scores the lower position is kept; the scores are the head sum
    of dot products and ignore the future."""
    L, hi, di, K_ = 30, 3, 5, 6
    QI, KI = _rand((L, hi, di), 70), _rand((L, di), 71)
    KI[10] = KI[4]                          # exact ties between positions 4 and 10
    KI[20] = KI[4]
    pos = np.arange(L)
    S = oracle.token_scores(QI, KI, pos)
    q, k = QI.double().numpy(), KI.double().numpy()
    for r in range(L):
        for u in range(L):
            want = -np.inf if u > r else sum(float(q[r, h] @ k[u]) for h in range(hi))
            assert S[r, u] == want or abs(S[r, u] - want) < 1e-12
    idx, gap = oracle.token_select(S, pos, K_)
    for r in range(L):
        kept = [int(u) for u in idx[r] if u >= 0]
        assert r in kept and len(kept) == min(K_, r + 1) and kept == sorted(kept)
        earlier = [u for u in kept if u != r]
        dropped = [u for u in range(r) if u not in kept]
        for a in earlier:
            for b in dropped:
                assert S[r, a] > S[r, b] or (S[r, a] == S[r, b] and a < b)
        if dropped and earlier:
            assert gap[r] == min(S[r, a] for a in earlier) - max(S[r, b] for b in dropped)
    # rows 21 and 25 have the cut inside the tied group: the lower positions stay
    for r in (21, 25):
        kept = set(int(u) for u in idx[r] if u >= 0)
        assert sorted(t for t in (4, 10, 20) if t in kept) == [4, 10]


def test_token_path_equals_block_path_on_constant_blocks():
    """Keys constant within each block, indexer = the group's query heads over
    the keys, query rows at block starts: the top (k-1) B earlier tokens are
    exactly the k-1 best blocks, so token attention (own position + those
    tokens) equals the block oracle's attention over its own selection."""
    B, nb, d, hq, hkv, k = 8, 9, 16, 4, 1, 4
    L = B * nb
    base = _rand((nb, hkv, d), 80)
    K = base.repeat_interleave(B, dim=0)               # [L, 1, d], constant per block
    Q, V = _rand((L, hq, d), 81), _rand((L, hkv, d), 82)
    pos = np.arange(B * (k - 1), L, B)                   # block starts with >= k-1 past blocks
    Qr = Q[pos]
    blk = oracle.forward(Qr, K, V, pos, B, k, 0.25)
    S = oracle.token_scores(Qr, K[:, 0], pos)
    idx, _ = oracle.token_select(S, pos, (k - 1) * B + 1)
    for r, t in enumerate(pos):
        past = sorted(int(j) for j in blk["idx"][r, 0] if 0 <= j < t // B)
        want = sorted([u for j in past for u in range(j * B, (j + 1) * B)] + [int(t)])
        assert [int(u) for u in idx[r] if u >= 0] == want
    O, lse = oracle.attend_tokens(Qr, K, V, pos, idx, 0.25)
    assert np.max(np.abs(O - blk["out"])) < 1e-12
    assert np.max(np.abs(lse - blk["lse"])) < 1e-12
