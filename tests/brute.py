"""Pure-Python brute force of shared-QK LSH attention, for tiny inputs only.

An independent restatement used to pin the float64 oracle: every quantity is
enumerated directly from its definition with Python floats and lists (no
NumPy arithmetic), so a dropped term, a wrong index or a transposed operand in
the oracle shows up as a mismatch.

Sources: Ultralytics glossary "Reformer", section "Atenção LSH" (bucket =
position of the largest value of [xR, -xR]; sort by bucket; equal blocks;
attend to own and previous block); twgreatdaily ICLR 2020 Reformer article,
section "1 LSH Attention" (sum over the admissible key set divided by its
partition function; Q = K with normalised keys; several rounds).
"""

from __future__ import annotations

import math


def dot(a, b):
    return sum(x * y for x, y in zip(a, b))


def brute_hash_row(x, R_round):
    """(bucket, top1, top2) of one row x (list of D floats) for one round.

    R_round is a D x (nb/2) nested list.  u lists p_0..p_{nb/2-1} and then
    -p_0..-p_{nb/2-1}; the bucket is the first index holding the maximum.
    """
    D = len(x)
    n = math.sqrt(dot(x, x))
    xh = [xi / n for xi in x] if n > 0 else [0.0] * D
    half = len(R_round[0])
    p = [sum(xh[d] * R_round[d][k] for d in range(D)) for k in range(half)]
    u = p + [-pk for pk in p]
    best = 0
    for j in range(1, len(u)):
        if u[j] > u[best]:
            best = j
    ordered = sorted(u, reverse=True)
    return best, ordered[0], ordered[1]


def admissible_slots(s, L, chunk, self_mask, perm=None, causal=False, bucket=None):
    """Sorted slots that the query at sorted slot s may attend to.

    Enumerated over every slot of the sequence: slot t is admissible when its
    chunk is the query's chunk or the one just before it (and, causal, when
    its original position perm[t] is not after the query's perm[s]; and, with
    bucket (by original position), when bucket[perm[t]] == bucket[perm[s]]).
    """
    k = s // chunk
    W = [t for t in range(L) if t // chunk == k or t // chunk == k - 1]
    if causal:
        W = [t for t in W if perm[t] <= perm[s]]
    if bucket is not None:
        W = [t for t in W if bucket[perm[t]] == bucket[perm[s]]]
    if self_mask and len(W) > 1:
        W = [t for t in W if t != s]
    return W


def brute_attend_round(qk, v, perm, chunk, self_mask, scale, causal=False, bucket=None,
                       all_buckets=None):
    """Per-position (o, lse) of one round, as dicts keyed by original position.

    qk, v: L lists of D floats; perm: list, perm[s] = original position.
    all_buckets (a list of every round's bucket list), when given: the weight
    of key j for query i is divided by the number of rounds in which
    all_buckets[r][j] == all_buckets[r][i].
    """
    L = len(perm)
    D = len(qk[0])
    out_o, out_lse = {}, {}
    for s in range(L):
        i = perm[s]
        logits = []
        for t in admissible_slots(s, L, chunk, self_mask, perm, causal, bucket):
            j = perm[t]
            nj = math.sqrt(dot(qk[j], qk[j]))
            lg = dot(qk[i], qk[j]) / nj * scale if nj > 0 else 0.0
            if all_buckets is not None:
                lg -= math.log(sum(1 for rb in all_buckets if rb[j] == rb[i]))
            logits.append((lg, j))
        Z = sum(math.exp(l) for l, _ in logits)
        out_o[i] = [sum(math.exp(l) * v[j][d] for l, j in logits) / Z for d in range(D)]
        out_lse[i] = math.log(Z)
    return out_o, out_lse


def brute_multiset_union(qk, v, perms, chunk, self_mask, scale):
    """Softmax over the multiset union of every round's admissible keys.

    A key admissible in several rounds is counted once per round.  Returns
    (o, lse) dicts keyed by original position.
    """
    L = len(perms[0])
    D = len(qk[0])
    terms = {i: [] for i in range(L)}
    for perm in perms:
        for s in range(L):
            i = perm[s]
            for t in admissible_slots(s, L, chunk, self_mask):
                j = perm[t]
                nj = math.sqrt(dot(qk[j], qk[j]))
                terms[i].append((dot(qk[i], qk[j]) / nj * scale if nj > 0 else 0.0, j))
    out_o, out_lse = {}, {}
    for i, tl in terms.items():
        Z = sum(math.exp(l) for l, _ in tl)
        out_o[i] = [sum(math.exp(l) * v[j][d] for l, j in tl) / Z for d in range(D)]
        out_lse[i] = math.log(Z)
    return out_o, out_lse


def brute_sort(bucket_row):
    """perm of one segment: positions ordered by the tuple (bucket, position)."""
    return [pos for _, pos in sorted((b, pos) for pos, b in enumerate(bucket_row))]
