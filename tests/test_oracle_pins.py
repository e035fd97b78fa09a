"""Pins of the float64 oracle against what the pages and the mathematics fix.

Runs on the CPU (``-m "not gpu"``).  Each test ties an oracle function to
something other than itself: the pages' worked example, a closed form, an
invariant, a textbook library routine, or a pure-Python brute force
(``tests/brute.py``).
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import (
    TIE_REL,
    oracle_attend,
    oracle_attend_slots,
    oracle_combine,
    oracle_hash,
    oracle_lsh_attention,
    oracle_sort,
)
from tests import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _pct_half_up(frac):
    return int(math.floor(100.0 * frac + 0.5))


# ---------------------------------------------------------------------------
# hash
# ---------------------------------------------------------------------------
def test_hash_collision_demo_matches_glossary_example():
    """Ultralytics glossary "Reformer", section "Atenção LSH": 72% / 9%."""
    with open(os.path.join(GOLDEN, "collision_demo.json")) as f:
        g = json.load(f)
    dim, nb, rounds = g["dim"], g["n_buckets"], g["rounds"]
    gen = torch.Generator().manual_seed(g["seed"])
    query = torch.randn(dim, generator=gen)
    near = query + 0.3 * torch.randn(dim, generator=gen)
    far = torch.randn(dim, generator=gen)
    R = torch.randn(rounds, dim, nb // 2, generator=gen)
    qk = torch.stack([query, near, far]).reshape(1, 1, 3, dim)
    buckets, _ = oracle_hash(qk, R, nb)
    b = buckets[0, 0]  # [rounds, 3]
    for col, name in ((1, "near"), (2, "far")):
        shared = float(np.mean(b[:, col] == b[:, 0]))
        assert _pct_half_up(shared) == g["printed"][name]["shared_bucket_pct"], (name, shared)
        cos = float(torch.nn.functional.cosine_similarity(query, qk[0, 0, col], dim=0))
        assert f"{cos:.2f}" == g["printed"][name]["cosine"]


def _orthonormal(D, n, seed):
    q, _ = np.linalg.qr(np.random.default_rng(seed).standard_normal((D, D)))
    return q[:, :n]


@pytest.mark.parametrize("D,nb", [(8, 8), (8, 16), (16, 8), (6, 12)])
def test_hash_orthonormal_columns_closed_form(D, nb):
    """x along column k of an orthonormal R gives p = e_k: bucket k; -x gives k + nb/2.

    With D == nb/2 the projection is square, so a transposed R fails here.
    """
    half = nb // 2
    Rr = _orthonormal(D, half, seed=D * 100 + nb)
    R = Rr[None]
    rows = []
    for k in range(half):
        rows.append(2.5 * Rr[:, k])
        rows.append(-0.7 * Rr[:, k])
    qk = np.array(rows)[None, None]
    buckets, near = oracle_hash(qk, R, nb)
    want = []
    for k in range(half):
        want += [k, k + half]
    assert buckets[0, 0, 0].tolist() == want
    assert not near.any()


def test_hash_near_tie_flag_threshold():
    """Two equal projections tie (flagged, lowest index wins); a gap just above 1e-5 is not flagged."""
    D, nb = 8, 8
    Rr = _orthonormal(D, nb // 2, seed=3)
    R = Rr[None]
    a, b = 1, 3
    rows = [Rr[:, a] + Rr[:, b],                         # exact tie
            Rr[:, a] + (1 - 2 * TIE_REL) * Rr[:, b],     # gap 2e-5: not a near tie
            Rr[:, a] + (1 - 0.5 * TIE_REL) * Rr[:, b],   # gap 5e-6: near tie
            -(Rr[:, b] + Rr[:, a])]                      # tie on the negative side
    buckets, near = oracle_hash(np.array(rows)[None, None], R, nb)
    assert buckets[0, 0, 0].tolist() == [a, a, a, a + nb // 2]
    assert near[0, 0, 0].tolist() == [True, False, True, True]


def test_hash_zero_vector_is_bucket0_and_flagged():
    R = np.random.default_rng(0).standard_normal((2, 4, 4))
    buckets, near = oracle_hash(np.zeros((1, 1, 1, 4)), R, 8)
    assert buckets.ravel().tolist() == [0, 0]
    assert near.all()


def test_hash_invariants_scale_negation_projection_scale():
    """h(a x) = h(x) (a > 0), h(-x) = (h(x) + nb/2) mod nb, h unchanged by R -> b R (b > 0)."""
    rng = np.random.default_rng(11)
    B, H, L, D, nb, nr = 2, 2, 64, 16, 32, 3
    x = rng.standard_normal((B, H, L, D))
    R = rng.standard_normal((nr, D, nb // 2))
    h0, f0 = oracle_hash(x, R, nb)
    alpha = rng.uniform(0.01, 100.0, size=(B, H, L, 1))
    h1, f1 = oracle_hash(alpha * x, R, nb)
    h2, f2 = oracle_hash(-x, R, nb)
    h3, f3 = oracle_hash(x, 7.25 * R, nb)
    ok = ~(f0 | f1 | f2 | f3)
    assert ok.mean() > 0.95
    assert np.array_equal(h1[ok], h0[ok])
    assert np.array_equal(h2[ok], ((h0 + nb // 2) % nb)[ok])
    assert np.array_equal(h3[ok], h0[ok])


def test_hash_matches_pure_python_enumeration():
    rng = np.random.default_rng(5)
    L, D, nb, nr = 20, 6, 10, 2
    x = rng.standard_normal((1, 1, L, D))
    R = rng.standard_normal((nr, D, nb // 2))
    h, f = oracle_hash(x, R, nb)
    for r in range(nr):
        Rl = R[r].tolist()
        for i in range(L):
            bk, u1, u2 = brute.brute_hash_row(x[0, 0, i].tolist(), Rl)
            assert h[0, 0, r, i] == bk
            assert f[0, 0, r, i] == ((u1 - u2) / max(abs(u1), 1e-30) < TIE_REL)


def test_hash_gaussian_marginal_is_uniform():
    """For any fixed x and R ~ N(0,1), x_hat @ R has iid N(0,1) entries, so every bucket is equally likely.

    One row hashed under many independent rounds gives iid bucket draws (chi-square against uniform).
    """
    from scipy import stats

    rng = np.random.default_rng(1)
    nb, D, rounds = 16, 32, 20000
    x = rng.standard_normal((1, 1, 1, D))
    R = rng.standard_normal((rounds, D, nb // 2))
    h, _ = oracle_hash(x, R, nb)
    counts = np.bincount(h.ravel(), minlength=nb)
    assert stats.chisquare(counts).pvalue > 1e-4, counts


def test_hash_collision_rate_rises_with_cosine():
    rng = np.random.default_rng(2)
    D, nb, rounds = 32, 16, 400
    q = rng.standard_normal(D)
    q /= np.linalg.norm(q)
    w = rng.standard_normal(D)
    w -= (w @ q) * q
    w /= np.linalg.norm(w)
    cosines = [0.0, 0.5, 0.8, 0.95, 0.99]
    vecs = [q] + [c * q + math.sqrt(1 - c * c) * w for c in cosines]
    R = rng.standard_normal((rounds, D, nb // 2))
    h, _ = oracle_hash(np.array(vecs)[None, None], R, nb)
    rates = [(h[0, 0, :, j + 1] == h[0, 0, :, 0]).mean() for j in range(len(cosines))]
    assert all(a < b for a, b in zip(rates, rates[1:])), rates


# ---------------------------------------------------------------------------
# sort
# ---------------------------------------------------------------------------
def test_sort_matches_tuple_sort_and_invariants():
    rng = np.random.default_rng(3)
    buckets = rng.integers(0, 7, size=(2, 3, 2, 50)).astype(np.int32)
    perm = oracle_sort(buckets)
    for idx in np.ndindex(*buckets.shape[:-1]):
        row = buckets[idx].tolist()
        p = perm[idx].tolist()
        assert p == brute.brute_sort(row)
        assert sorted(p) == list(range(50))
        keys = [(row[i], i) for i in p]
        assert keys == sorted(keys)


def test_sort_skewed_single_bucket_is_identity():
    b = np.full((1, 1, 1, 300), 5, dtype=np.int32)
    assert oracle_sort(b)[0, 0, 0].tolist() == list(range(300))


# ---------------------------------------------------------------------------
# attend
# ---------------------------------------------------------------------------
def _random_perm(rng, L, nr):
    return np.stack([rng.permutation(L) for _ in range(nr)]).astype(np.int32)


@pytest.mark.parametrize("L,chunk,self_mask", [
    (24, 4, True), (24, 4, False), (16, 1, True), (16, 16, True), (16, 8, True),
    (12, 3, False), (8, 1, False),
])
def test_attend_matches_admissible_set_enumeration(L, chunk, self_mask):
    rng = np.random.default_rng(L * 31 + chunk)
    D, nr = 5, 2
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    perm = _random_perm(rng, L, nr)[None, None]
    scale = 0.37
    o, lse = oracle_attend(qk, v, perm, chunk, self_mask, scale)
    for r in range(nr):
        bo, bl = brute.brute_attend_round(qk[0, 0].tolist(), v[0, 0].tolist(),
                                          perm[0, 0, r].tolist(), chunk, self_mask, scale)
        for i in range(L):
            assert np.allclose(o[0, 0, r, i], bo[i], rtol=0, atol=1e-12)
            assert abs(lse[0, 0, r, i] - bl[i]) < 1e-12


@pytest.mark.parametrize("self_mask", [True, False])
def test_attend_single_chunk_equals_dense_softmax(self_mask):
    """chunk == L: every round is full softmax attention with normalised keys (and the self mask)."""
    rng = np.random.default_rng(9)
    B, H, L, D, nr = 2, 2, 32, 8, 3
    qk = rng.standard_normal((B, H, L, D))
    v = rng.standard_normal((B, H, L, D))
    perm = np.stack([np.stack([_random_perm(rng, L, nr) for _ in range(H)]) for _ in range(B)])
    o, lse = oracle_attend(qk, v, perm, L, self_mask)
    scale = 1 / math.sqrt(D)
    for b in range(B):
        for h in range(H):
            x = qk[b, h]
            kh = x / np.linalg.norm(x, axis=1, keepdims=True)
            S = (x @ kh.T) * scale
            if self_mask:
                np.fill_diagonal(S, -np.inf)
            Z = np.exp(S).sum(1)
            dense = (np.exp(S) / Z[:, None]) @ v[b, h]
            for r in range(nr):
                assert np.allclose(o[b, h, r], dense, atol=1e-12)
                assert np.allclose(lse[b, h, r], np.log(Z), atol=1e-12)
    out, big = oracle_combine(o, lse)
    assert np.allclose(out, o[:, :, 0], atol=1e-12)
    assert np.allclose(big, lse[:, :, 0] + math.log(nr), atol=1e-12)


def test_attend_convexity_and_constant_values():
    rng = np.random.default_rng(4)
    L, D, chunk = 64, 6, 8
    qk = rng.standard_normal((1, 1, L, D))
    perm = _random_perm(rng, L, 1)[None, None]
    o1, _ = oracle_attend(qk, np.ones((1, 1, L, D)), perm, chunk)
    assert np.allclose(o1, 1.0, atol=1e-12)
    v = rng.standard_normal((1, 1, L, D))
    o, _ = oracle_attend(qk, v, perm, chunk)
    p = perm[0, 0, 0]
    for s in range(L):
        W = brute.admissible_slots(s, L, chunk, True)
        vals = v[0, 0, p[W]]
        assert np.all(o[0, 0, 0, p[s]] <= vals.max(0) + 1e-12)
        assert np.all(o[0, 0, 0, p[s]] >= vals.min(0) - 1e-12)


def test_attend_chunk1_self_only_fallback():
    """chunk 1: slot 0 has only itself (o = v_i, lse = |q_i| * scale); slot s > 0 sees only slot s-1."""
    rng = np.random.default_rng(6)
    L, D = 6, 4
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    perm = _random_perm(rng, L, 1)[None, None]
    scale = 0.5
    o, lse = oracle_attend(qk, v, perm, 1, True, scale)
    p = perm[0, 0, 0]
    i0 = p[0]
    assert np.allclose(o[0, 0, 0, i0], v[0, 0, i0])
    assert abs(lse[0, 0, 0, i0] - np.linalg.norm(qk[0, 0, i0]) * scale) < 1e-12
    for s in range(1, L):
        i, j = p[s], p[s - 1]
        assert np.allclose(o[0, 0, 0, i], v[0, 0, j])
        want = qk[0, 0, i] @ qk[0, 0, j] / np.linalg.norm(qk[0, 0, j]) * scale
        assert abs(lse[0, 0, 0, i] - want) < 1e-12


def test_attend_two_chunks_first_chunk_self_contained():
    """L / chunk == 2: chunk 0 does not wrap around to chunk 1."""
    rng = np.random.default_rng(8)
    L, D, chunk = 8, 3, 4
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    perm = _random_perm(rng, L, 1)[None, None]
    o, _ = oracle_attend(qk, v, perm, chunk)
    v2 = v.copy()
    v2[0, 0, perm[0, 0, 0, chunk:]] += 100.0  # change every value of chunk 1
    o2, _ = oracle_attend(qk, v2, perm, chunk)
    first = perm[0, 0, 0, :chunk]
    assert np.allclose(o[0, 0, 0, first], o2[0, 0, 0, first], atol=1e-12)


def test_attend_slots_matches_full():
    rng = np.random.default_rng(12)
    L, D, chunk = 64, 5, 8
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    perm = _random_perm(rng, L, 1)[None, None]
    o, lse = oracle_attend(qk, v, perm, chunk)
    slots = [0, 7, 8, 33, 63]
    pos, os_, ls = oracle_attend_slots(qk[0, 0], v[0, 0], perm[0, 0, 0], chunk, slots)
    assert pos.tolist() == perm[0, 0, 0, slots].tolist()
    assert np.allclose(os_, o[0, 0, 0, pos], atol=0)
    assert np.allclose(ls, lse[0, 0, 0, pos], atol=0)


# ---------------------------------------------------------------------------
# combine and end to end
# ---------------------------------------------------------------------------
def test_combine_equals_softmax_over_multiset_union():
    rng = np.random.default_rng(13)
    L, D, chunk, nr = 16, 4, 4, 3
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    perm = _random_perm(rng, L, nr)[None, None]
    scale = 0.8
    o, lse = oracle_attend(qk, v, perm, chunk, True, scale)
    out, big = oracle_combine(o, lse)
    bo, bl = brute.brute_multiset_union(qk[0, 0].tolist(), v[0, 0].tolist(),
                                        [perm[0, 0, r].tolist() for r in range(nr)], chunk, True, scale)
    for i in range(L):
        assert np.allclose(out[0, 0, i], bo[i], atol=1e-12)
        assert abs(big[0, 0, i] - bl[i]) < 1e-12


def test_combine_identical_rounds_collapse():
    rng = np.random.default_rng(14)
    o1 = rng.standard_normal((2, 1, 1, 10, 3))
    l1 = rng.standard_normal((2, 1, 1, 10))
    o = np.repeat(o1, 4, axis=2)
    l = np.repeat(l1, 4, axis=2)
    out, big = oracle_combine(o, l)
    assert np.allclose(out, o1[:, :, 0], atol=1e-12)
    assert np.allclose(big, l1[:, :, 0] + math.log(4), atol=1e-12)


def test_end_to_end_matches_brute_force_pipeline():
    rng = np.random.default_rng(21)
    L, D, nb, chunk, nr = 24, 4, 6, 4, 2
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    R = rng.standard_normal((nr, D, nb // 2))
    res = oracle_lsh_attention(qk, v, R, nb, chunk)
    X = qk[0, 0].tolist()
    perms = []
    for r in range(nr):
        bk = [brute.brute_hash_row(X[i], R[r].tolist())[0] for i in range(L)]
        assert bk == res["buckets"][0, 0, r].tolist()
        perms.append(brute.brute_sort(bk))
    assert [p for p in perms] == [res["perm"][0, 0, r].tolist() for r in range(nr)]
    bo, bl = brute.brute_multiset_union(X, v[0, 0].tolist(), perms, chunk, True, 1 / math.sqrt(D))
    for i in range(L):
        assert np.allclose(res["out"][0, 0, i], bo[i], atol=1e-12)
        assert abs(res["lse"][0, 0, i] - bl[i]) < 1e-12


# ---------------------------------------------------------------- causal variant
@pytest.mark.parametrize("L,chunk,self_mask", [(24, 4, True), (24, 4, False), (16, 16, True), (12, 3, True),
                                               (8, 1, True)])
def test_attend_causal_matches_admissible_set_enumeration(L, chunk, self_mask):
    """causal: keys after the query's original position are not admissible (brute force)."""
    rng = np.random.default_rng(L * 17 + chunk)
    D, nr = 5, 2
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    perm = _random_perm(rng, L, nr)[None, None]
    scale = 0.41
    o, lse = oracle_attend(qk, v, perm, chunk, self_mask, scale, causal=True)
    for r in range(nr):
        bo, bl = brute.brute_attend_round(qk[0, 0].tolist(), v[0, 0].tolist(), perm[0, 0, r].tolist(), chunk,
                                          self_mask, scale, causal=True)
        for i in range(L):
            assert np.allclose(o[0, 0, r, i], bo[i], rtol=0, atol=1e-12)
            assert abs(lse[0, 0, r, i] - bl[i]) < 1e-12


def test_attend_causal_single_chunk_equals_dense_causal_softmax():
    """chunk == L, causal: dense attention of position i over positions j < i (normalised keys);
    position 0 has no earlier key and sees only itself, whatever the permutation."""
    rng = np.random.default_rng(21)
    L, D, nr = 24, 6, 3
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    perm = _random_perm(rng, L, nr)[None, None]
    o, lse = oracle_attend(qk, v, perm, L, True, causal=True)
    x = qk[0, 0]
    kh = x / np.linalg.norm(x, axis=1, keepdims=True)
    S = (x @ kh.T) / math.sqrt(D)
    S[np.triu_indices(L, 0)] = -np.inf          # keys j >= i out (self too)
    S[0, 0] = x[0] @ kh[0] / math.sqrt(D)       # position 0: only itself
    Z = np.exp(S).sum(1)
    dense = (np.exp(S) / Z[:, None]) @ v[0, 0]
    for r in range(nr):
        assert np.allclose(o[0, 0, r], dense, atol=1e-12)
        assert np.allclose(lse[0, 0, r], np.log(Z), atol=1e-12)
    assert np.allclose(o[0, 0, 0, 0], v[0, 0, 0])


def test_attend_causal_constant_values_and_future_independence():
    """V == 1 gives 1; changing only the rows of positions after i leaves position i unchanged
    in a single-chunk window (causal), while it does change without the mask."""
    rng = np.random.default_rng(23)
    L, D = 16, 4
    qk = rng.standard_normal((1, 1, L, D))
    perm = _random_perm(rng, L, 1)[None, None]
    o1, _ = oracle_attend(qk, np.ones((1, 1, L, D)), perm, 8, causal=True)
    assert np.allclose(o1, 1.0, atol=1e-12)
    v = rng.standard_normal((1, 1, L, D))
    o, _ = oracle_attend(qk, v, perm, L, causal=True)
    i = 9
    qk2, v2 = qk.copy(), v.copy()
    qk2[0, 0, i + 1:] += rng.standard_normal((L - i - 1, D))
    v2[0, 0, i + 1:] += 5.0
    o2, _ = oracle_attend(qk2, v2, perm, L, causal=True)
    assert np.allclose(o[0, 0, 0, :i + 1], o2[0, 0, 0, :i + 1], atol=1e-12)
    o3, _ = oracle_attend(qk, v, perm, L, causal=False)
    o4, _ = oracle_attend(qk2, v2, perm, L, causal=False)
    assert not np.allclose(o3[0, 0, 0, i], o4[0, 0, 0, i])


# ------------------------------------------------- bucket-equality mask and union
def _bucketed(rng, L, nr, nb, sorted_perm):
    """Random buckets [nr, L] and a permutation per round: the stable sort by
    bucket when sorted_perm, else an unrelated random permutation."""
    bk = rng.integers(0, nb, size=(nr, L)).astype(np.int32)
    if sorted_perm:
        perm = np.stack([np.argsort(bk[r], kind="stable") for r in range(nr)]).astype(np.int32)
    else:
        perm = _random_perm(rng, L, nr)
    return bk, perm


@pytest.mark.parametrize("L,chunk,self_mask,causal,union,sorted_perm", [
    (24, 4, True, False, False, True), (24, 4, False, False, False, False), (16, 16, True, False, False, True),
    (12, 3, True, True, False, True), (8, 1, True, False, False, True), (24, 4, True, False, True, True),
    (24, 6, True, True, True, False), (16, 8, False, False, True, True),
])
def test_attend_bucket_mask_matches_admissible_set_enumeration(L, chunk, self_mask, causal, union, sorted_perm):
    """bucket mask: a key outside the query's bucket is not admissible; union: each logit is
    lowered by log(#rounds sharing the bucket) (brute force over the admissible slots)."""
    rng = np.random.default_rng(L * 13 + chunk * 3 + union)
    D, nr, nb = 5, 3, 3
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    bk, perm = _bucketed(rng, L, nr, nb, sorted_perm)
    scale = 0.53
    o, lse = oracle_attend(qk, v, perm[None, None], chunk, self_mask, scale, causal=causal,
                           buckets=bk[None, None], union=union)
    allb = [bk[r].tolist() for r in range(nr)] if union else None
    for r in range(nr):
        bo, bl = brute.brute_attend_round(qk[0, 0].tolist(), v[0, 0].tolist(), perm[r].tolist(), chunk,
                                          self_mask, scale, causal=causal, bucket=bk[r].tolist(),
                                          all_buckets=allb)
        for i in range(L):
            assert np.allclose(o[0, 0, r, i], bo[i], rtol=0, atol=1e-12)
            assert abs(lse[0, 0, r, i] - bl[i]) < 1e-12


def _dense_logits(x, D):
    kh = x / np.linalg.norm(x, axis=1, keepdims=True)
    return (x @ kh.T) / math.sqrt(D)


def test_attend_bucket_mask_single_chunk_equals_dense_same_bucket_softmax():
    """chunk == L, bucket mask: round r is dense attention of i over the other members of its
    bucket b_r(i); a query alone in its bucket sees only itself."""
    rng = np.random.default_rng(31)
    L, D, nr, nb = 24, 6, 3, 5
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    bk, perm = _bucketed(rng, L, nr, nb, True)
    bk[0, 7] = nb  # position 7 alone in its bucket in round 0
    perm[0] = np.argsort(bk[0], kind="stable")
    o, lse = oracle_attend(qk, v, perm[None, None], L, True, buckets=bk[None, None])
    S0 = _dense_logits(qk[0, 0], D)
    for r in range(nr):
        S = S0.copy()
        same = bk[r][:, None] == bk[r][None, :]
        alone = same.sum(1) == 1
        S[~same] = -np.inf
        S[np.diag_indices(L)] = np.where(alone, np.diag(S0), -np.inf)
        Z = np.exp(S).sum(1)
        assert np.allclose(o[0, 0, r], (np.exp(S) / Z[:, None]) @ v[0, 0], atol=1e-12)
        assert np.allclose(lse[0, 0, r], np.log(Z), atol=1e-12)
    assert np.allclose(o[0, 0, 0, 7], v[0, 0, 7])


def test_union_single_chunk_merge_equals_softmax_over_set_union():
    """chunk == L, bucket mask and union, no query alone in any round: the rounds merged by
    their log-sum-exp give softmax attention over U_i = {j != i : b_r(j) == b_r(i) for some r},
    each key once; the plain merge (no correction) does not."""
    rng = np.random.default_rng(37)
    L, D, nr, nb = 32, 5, 4, 3
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    bk, perm = _bucketed(rng, L, nr, nb, True)
    for r in range(nr):
        assert np.all(np.bincount(bk[r], minlength=nb) >= 2)  # nobody alone
    o, lse = oracle_attend(qk, v, perm[None, None], L, True, buckets=bk[None, None], union=True)
    out, big = oracle_combine(o, lse)
    S = _dense_logits(qk[0, 0], D)
    U = np.zeros((L, L), dtype=bool)
    for r in range(nr):
        U |= bk[r][:, None] == bk[r][None, :]
    np.fill_diagonal(U, False)
    assert not np.all(U)  # the union is a proper subset of the sequence
    S[~U] = -np.inf
    Z = np.exp(S).sum(1)
    assert np.allclose(out[0, 0], (np.exp(S) / Z[:, None]) @ v[0, 0], atol=1e-12)
    assert np.allclose(big[0, 0], np.log(Z), atol=1e-12)
    o2, lse2 = oracle_attend(qk, v, perm[None, None], L, True, buckets=bk[None, None], union=False)
    out2, _ = oracle_combine(o2, lse2)
    assert not np.allclose(out2[0, 0], out[0, 0], atol=1e-6)


def test_union_identical_rounds_collapse_to_one_round():
    """n identical rounds with the union correction: every pair shares all n, so each round's
    lse is the single round's minus log n and the merged LSE equals the single round's."""
    rng = np.random.default_rng(41)
    L, D, chunk, n = 24, 4, 6, 4
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    bk1, perm1 = _bucketed(rng, L, 1, 3, True)
    bk, perm = np.repeat(bk1, n, axis=0), np.repeat(perm1, n, axis=0)
    o1, l1 = oracle_attend(qk, v, perm1[None, None], chunk, True, buckets=bk1[None, None])
    o, lse = oracle_attend(qk, v, perm[None, None], chunk, True, buckets=bk[None, None], union=True)
    assert np.allclose(lse, l1 - math.log(n), atol=1e-12)
    out, big = oracle_combine(o, lse)
    assert np.allclose(out, o1[:, :, 0], atol=1e-12)
    assert np.allclose(big, l1[:, :, 0], atol=1e-12)


def test_union_needs_bucket_mask():
    qk = np.ones((1, 1, 4, 2))
    with pytest.raises(ValueError):
        oracle_attend(qk, qk, np.zeros((1, 1, 1, 4), dtype=np.int32) + np.arange(4), 2, union=True)


def test_bucket_mask_end_to_end_matches_brute_force_pipeline():
    """hash -> sort -> bucket-masked attention with the union correction, brute force per round."""
    rng = np.random.default_rng(43)
    L, D, nb, chunk, nr = 24, 4, 4, 4, 3
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    R = rng.standard_normal((nr, D, nb // 2))
    res = oracle_lsh_attention(qk, v, R, nb, chunk, bucket_mask=True, union=True)
    X = qk[0, 0].tolist()
    bks = [[brute.brute_hash_row(X[i], R[r].tolist())[0] for i in range(L)] for r in range(nr)]
    for r in range(nr):
        assert bks[r] == res["buckets"][0, 0, r].tolist()
        perm = brute.brute_sort(bks[r])
        bo, bl = brute.brute_attend_round(X, v[0, 0].tolist(), perm, chunk, True, 1 / math.sqrt(D),
                                          bucket=bks[r], all_buckets=bks)
        for i in range(L):
            assert np.allclose(res["o_rounds"][0, 0, r, i], bo[i], atol=1e-12)
            assert abs(res["lse_rounds"][0, 0, r, i] - bl[i]) < 1e-12
