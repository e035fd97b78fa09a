"""Float64 CPU oracle of shared-QK LSH attention, forward pass.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Slow on purpose: plain
NumPy in float64 on the exact input values, one step of the method at a time,
no blocking, fusion or reordering beyond what the method itself states.

Sources (the pages this follows, by title and section):

* [GLOSSARY] Ultralytics glossary page "Reformer" (pt), section "Atenção LSH":
  one shared projection for queries and keys; angular LSH: multiply by a random
  matrix R and take as bucket the position of the largest value of [xR, -xR];
  sort tokens by bucket, split the sorted sequence into equal blocks, each
  token attends to its own block and the previous one; several hashing rounds
  run in parallel.  Its worked example (d=64, 16 buckets, 1000 rounds, seed 0:
  72% / 9% shared buckets at cosine 0.96 / 0.04) pins ``oracle_hash``.
* [ZH-ICLR] twgreatdaily.com article on the ICLR 2020 oral "Reformer: The
  Efficient Transformer", section "1 LSH Attention": attention of query i as a
  sum over an admissible key set P_i normalised by a partition function; keys
  outside the set are masked; Q = K with keys length-normalised; two-level
  sort by (bucket, position inside the bucket); consecutive equal chunks where
  a later chunk looks back one chunk; several hash rounds combined.
* [JA-SCHOLAR] ai-scholar.tech article "計算時間とメモリの壁を打破！
  Transformerの次世代モデルReformer", sections "Transformerの問題点とは"
  (scaled dot product, 1/sqrt(d_k)) and "LSH Attention" (bucket, sort, equal
  chunks, attend to own and previous chunk).
* [RU-VIDEO] rdly.ru summary "Как уместить 64 000 токенов в одну видеокарту",
  section "Разделение на блоки (Chunking)": fixed-size blocks of the sorted
  sequence, each element attends inside its block and the neighbouring one.

Readings where the pages are silent or garbled:

* chunk 0 has no previous chunk (no wrap-around); the window is a *set* of
  sorted slots, so a single chunk covering the sequence is not duplicated;
* no bucket-equality mask inside the window: every key of the two chunks is
  admissible;
* queries stay raw, keys are unit-normalised, logit scale defaults to
  1/sqrt(D);
* a token does not attend to itself unless it is the only key in its window;
* bucket-equality variant (twgreatdaily article, "1 LSH Attention": the
  admissible set of a query is the keys of its own bucket, batched by chunks):
  inside the chunk window a key is admissible only when it shares the query's
  bucket in that round; the self rule then applies to what remains;
* multi-round union variant (twgreatdaily article, "1 LSH Attention": the
  admissible set over several rounds is the union of the rounds' sets, with a
  per-pair correction whose formula the page lost in extraction): read as the
  original paper's duplicate count, each admissible logit of a round is lowered
  by log N_ij, N_ij = the number of rounds whose hash puts i and j in the same
  bucket (the self pair shares every round); used with the bucket-equality
  mask, the log-sum-exp merge then counts each key of the union once whenever
  each shared bucket lies inside the query's window;
* causal variant (the pages' character-level language model, ai-scholar.tech
  article, results on enwik8-64K; masking in the twgreatdaily article, "1 LSH
  Attention"): a key whose original position is after the query's is not
  admissible; the self rule then applies to what remains, so a query with no
  earlier key in its window sees only itself;
* rounds are merged by their per-query log-sum-exp weights;
* argmax ties go to the lowest index; a hash is "near-tie" when the top two
  values of [p, -p] differ by less than ``TIE_REL`` relative to the top.
"""

from __future__ import annotations

import math

import numpy as np

TIE_REL = 1e-5  # relative top-1 / top-2 gap below which a hash counts as a near tie


def _f64(a) -> np.ndarray:
    """Exact float64 copy of an array (bf16 / f32 values are representable)."""
    if hasattr(a, "detach"):  # a torch tensor: widen on the CPU, exactly
        import torch

        a = a.detach().to("cpu", torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------
# a1  hash  [GLOSSARY "Atenção LSH"]; [ZH-ICLR §1]; [JA-SCHOLAR "LSH Attention"]
# ----------------------------------------------------------------------------
def oracle_hash(qk, R, n_buckets: int, tie_rel: float = TIE_REL, row_block: int = 8192):
    """Angular LSH bucket of every shared query/key row, for every round.

    qk: [B, H, L, D]; R: [n_rounds, D, n_buckets // 2] (one random projection
    per round, shared by all batches and heads).

    For each row x and round r: x_hat = x / ||x||, p = x_hat @ R[r]
    (n_buckets/2 values), u = [p, -p] (n_buckets values, first half from p),
    bucket = index of the largest entry of u (lowest index on exact ties).
    near_tie = (u1 - u2) / |u1| < tie_rel with u1 >= u2 the two largest
    entries of u counted as a multiset.

    Returns (buckets int32 [B, H, n_rounds, L], near_tie bool [B, H, n_rounds, L]).
    """
    x = _f64(qk)
    Rm = _f64(R)
    B, H, L, D = x.shape
    n_rounds, D2, half = Rm.shape
    if D2 != D or 2 * half != n_buckets:
        raise ValueError("R must be [n_rounds, D, n_buckets // 2]")
    rows = x.reshape(B * H * L, D)
    norms = np.sqrt(np.sum(rows * rows, axis=1, keepdims=True))
    x_hat = rows / np.maximum(norms, 1e-12)
    buckets = np.empty((B * H * L, n_rounds), dtype=np.int32)
    near = np.empty((B * H * L, n_rounds), dtype=bool)
    for r in range(n_rounds):
        for lo in range(0, B * H * L, row_block):
            p = x_hat[lo:lo + row_block] @ Rm[r]
            u = np.concatenate([p, -p], axis=1)
            buckets[lo:lo + row_block, r] = np.argmax(u, axis=1)  # first maximum
            top2 = np.partition(u, n_buckets - 2, axis=1)[:, n_buckets - 2:]
            u2, u1 = top2[:, 0], top2[:, 1]
            near[lo:lo + row_block, r] = (u1 - u2) / np.maximum(np.abs(u1), 1e-30) < tie_rel
    buckets = buckets.reshape(B, H, L, n_rounds).transpose(0, 1, 3, 2).copy()
    near = near.reshape(B, H, L, n_rounds).transpose(0, 1, 3, 2).copy()
    return buckets, near


# ----------------------------------------------------------------------------
# a2  sort  [ZH-ICLR §1: two-level sort by bucket, then position in bucket];
#           [JA-SCHOLAR "LSH Attention"]; [GLOSSARY "Atenção LSH"]
# ----------------------------------------------------------------------------
def oracle_sort(buckets):
    """perm[..., s] = original position of sorted slot s, per (b, h, round).

    Tokens are ordered by the key (bucket, position): np.lexsort with the
    position as the minor key and the bucket as the major key.
    """
    b = np.asarray(buckets)
    L = b.shape[-1]
    flat = b.reshape(-1, L)
    pos = np.arange(L)
    perm = np.empty(flat.shape, dtype=np.int32)
    for seg in range(flat.shape[0]):
        perm[seg] = np.lexsort((pos, flat[seg]))
    return perm.reshape(b.shape)


# ----------------------------------------------------------------------------
# a3 + a4  gather and chunk attention
#   [ZH-ICLR §1: per-query sum over the admissible set with its partition
#    function, masked keys, Q = K with normalised keys, later chunk looks back
#    one chunk]; [JA-SCHOLAR "Transformerの問題点とは": 1/sqrt(d_k)];
#   [RU-VIDEO "Разделение на блоки"]; [GLOSSARY "Atenção LSH"]
# ----------------------------------------------------------------------------
def _window_slots(k: int, chunk: int) -> np.ndarray:
    """Sorted slots visible to chunk k: chunk k-1 (if it exists) and chunk k."""
    return np.arange(max(k - 1, 0) * chunk, (k + 1) * chunk)


def _chunk_logits(x, k_hat, perm_seg, k, chunk, self_mask, scale, causal=False, bucket_seg=None,
                  union_buckets=None):
    """Logits of the queries of sorted chunk k against its window, -inf where not admissible.

    Returns (qi [c] original positions of the queries, kj [|W|] of the keys, logits [c, |W|]).

    causal: a key whose original position is after the query's is not
    admissible (the language-model reading of the window).  bucket_seg (the
    round's bucket of every original position), when given: a key in another
    bucket than the query's is not admissible.  The self entry is dropped while
    the query has another admissible key.  union_buckets ([n_rounds, L], every
    round's bucket by original position), when given: each admissible logit is
    lowered by log N, N = the number of rounds whose hash puts query and key in
    the same bucket (the self pair: every round).
    """
    q_slots = np.arange(k * chunk, (k + 1) * chunk)
    w_slots = _window_slots(k, chunk)
    qi = perm_seg[q_slots]
    kj = perm_seg[w_slots]
    logits = (x[qi] @ k_hat[kj].T) * scale  # [c, |W|]
    adm = np.ones(logits.shape, dtype=bool)
    if causal:
        adm &= kj[None, :] <= qi[:, None]
    if bucket_seg is not None:
        adm &= bucket_seg[kj][None, :] == bucket_seg[qi][:, None]
    if self_mask:
        is_self = q_slots[:, None] == w_slots[None, :]
        others = np.any(adm & ~is_self, axis=1, keepdims=True)
        adm &= ~(is_self & others)
    if union_buckets is not None:
        ub = np.asarray(union_buckets)
        n_shared = np.sum(ub[:, kj][:, None, :] == ub[:, qi][:, :, None], axis=0)  # [c, |W|]
        logits[adm] -= np.log(n_shared[adm])
    logits[~adm] = -np.inf
    return qi, kj, logits


def _attend_chunk(x, k_hat, v, perm_seg, k, chunk, self_mask, scale, causal=False, bucket_seg=None,
                  union_buckets=None):
    """Outputs of the queries of sorted chunk k of one (b, h, round) segment (masks as in
    ``_chunk_logits``).  Returns (orig positions [c], o [c, D], lse [c])."""
    qi, kj, logits = _chunk_logits(x, k_hat, perm_seg, k, chunk, self_mask, scale, causal, bucket_seg,
                                   union_buckets)
    m = np.max(logits, axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.sum(np.exp(logits - m), axis=1))
    weights = np.exp(logits - lse[:, None])
    return qi, weights @ v[kj], lse


def _prep_slice(qk_bh, v_bh):
    x = _f64(qk_bh)
    vv = _f64(v_bh)
    norms = np.sqrt(np.sum(x * x, axis=1, keepdims=True))
    return x, x / np.maximum(norms, 1e-12), vv


def oracle_attend(qk, v, perm, chunk: int, self_mask: bool = True, scale: float | None = None,
                  causal: bool = False, buckets=None, union: bool = False):
    """Per-round LSH attention outputs in original token order.

    qk, v: [B, H, L, D]; perm: [B, H, n_rounds, L].  causal: keys after the
    query's position are not admissible.  buckets ([B, H, n_rounds, L], by
    original position), when given: keys outside the query's bucket are not
    admissible (the pages' bucket-equality mask inside the window).  union
    (needs buckets): every admissible logit is lowered by the log of the number
    of rounds in which query and key share a bucket, so that the rounds merged
    by their log-sum-exp count each shared key once.
    Returns (o [B, H, n_rounds, L, D] float64, lse [B, H, n_rounds, L] float64).
    """
    B, H, L, D = qk.shape
    perm = np.asarray(perm)
    n_rounds = perm.shape[2]
    if L % chunk:
        raise ValueError("L must be a multiple of chunk")
    if union and buckets is None:
        raise ValueError("the union correction needs the bucket-equality mask")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    bk = None if buckets is None else np.asarray(buckets)
    o = np.empty((B, H, n_rounds, L, D))
    lse = np.empty((B, H, n_rounds, L))
    for b in range(B):
        for h in range(H):
            x, k_hat, vv = _prep_slice(qk[b, h], v[b, h])
            for r in range(n_rounds):
                for k in range(L // chunk):
                    qi, ob, lb = _attend_chunk(x, k_hat, vv, perm[b, h, r], k, chunk, self_mask, scale, causal,
                                               None if bk is None else bk[b, h, r],
                                               bk[b, h] if union else None)
                    o[b, h, r, qi] = ob
                    lse[b, h, r, qi] = lb
    return o, lse


def oracle_attend_slots(qk_bh, v_bh, perm_seg, chunk: int, slots, self_mask: bool = True,
                        scale: float | None = None, causal: bool = False, bucket_seg=None,
                        union_buckets=None):
    """Outputs of selected sorted slots of ONE (b, h, round) segment.

    For checks at sizes where a whole segment is too slow: qk_bh, v_bh are
    [L, D]; perm_seg is [L]; slots are sorted-slot indices.  The chunk of each
    slot is evaluated in full and the requested rows are returned.  bucket_seg
    ([L], this round's buckets) and union_buckets ([n_rounds, L], every round's)
    select the bucket-equality mask and the union correction.

    Returns (orig positions [n], o [n, D], lse [n]).
    """
    L, D = qk_bh.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    x, k_hat, vv = _prep_slice(qk_bh, v_bh)
    slots = np.asarray(slots)
    out_pos = np.empty(len(slots), dtype=np.int64)
    out_o = np.empty((len(slots), D))
    out_l = np.empty(len(slots))
    cache = {}
    for n, s in enumerate(slots):
        k = int(s) // chunk
        if k not in cache:
            cache[k] = _attend_chunk(x, k_hat, vv, np.asarray(perm_seg), k, chunk, self_mask, scale, causal,
                                     None if bucket_seg is None else np.asarray(bucket_seg), union_buckets)
        qi, ob, lb = cache[k]
        j = int(s) - k * chunk
        out_pos[n], out_o[n], out_l[n] = qi[j], ob[j], lb[j]
    return out_pos, out_o, out_l


# ----------------------------------------------------------------------------
# a5  combine rounds  [ZH-ICLR §1: several hash rounds, each with its own
#      admissible set]; [GLOSSARY "Atenção LSH": rounds run in parallel];
#      merged by per-query log-sum-exp weights
# ----------------------------------------------------------------------------
def oracle_combine(o, lse):
    """out = sum_r w_r * o_r with w_r = exp(lse_r - LSE), LSE = log sum_r exp(lse_r).

    o: [B, H, n_rounds, L, D]; lse: [B, H, n_rounds, L].
    Returns (out [B, H, L, D], LSE [B, H, L]).
    """
    o = _f64(o)
    lse = _f64(lse)
    m = np.max(lse, axis=2, keepdims=True)
    big = m[:, :, 0] + np.log(np.sum(np.exp(lse - m), axis=2))
    w = np.exp(lse - big[:, :, None, :])
    out = np.sum(w[..., None] * o, axis=2)
    return out, big


# ----------------------------------------------------------------------------
# backward  [the forward above, differentiated by the chain rule with the hash,
#            the sort and the masks held fixed (a bucket is a piecewise-constant
#            function of x); GLOSSARY / ZH-ICLR: training through LSH attention
#            recomputes from the stored buckets]
# ----------------------------------------------------------------------------
def oracle_attend_backward(qk, v, perm, chunk: int, dout, self_mask: bool = True, scale: float | None = None,
                           causal: bool = False, buckets=None, union: bool = False):
    """Gradients (dqk, dv) [B, H, L, D] float64 of sum(dout * out) for the merged output.

    The forward is recomputed here: per-round (o_r, lse_r), then out and LSE.  Chain rule:

      merge: out = sum_r w_r o_r, w_r = exp(lse_r - LSE)
             d o_r = w_r dout;  d lse_r = w_r (dout . o_r - dout . out)
      round: o = sum_j p_j v_j, p_j = exp(z_j - lse), lse = log sum_j exp(z_j)
             d v_j += p_j d o;  d z_j = p_j (d o . v_j - d o . o) + p_j d lse
      logit: z_ij = scale * x_i . k_j (less log N under the union correction, a constant),
             k_j = x_j / max(||x_j||, 1e-12)
             d x_i += scale * sum_j dz_ij k_j                          (query role)
             d k_j  = scale * sum_i dz_ij x_i
             d x_j += (d k_j - (d k_j . k_j) k_j) / ||x_j||            (key role; the clamp's
                      linear branch d k_j / 1e-12 when ||x_j|| < 1e-12)
    """
    qk = _f64(qk)
    v = _f64(v)
    dout = _f64(dout)
    B, H, L, D = qk.shape
    perm = np.asarray(perm)
    n_rounds = perm.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o, lse = oracle_attend(qk, v, perm, chunk, self_mask, scale, causal, buckets, union)
    out, big = oracle_combine(o, lse)
    w = np.exp(lse - big[:, :, None, :])                                    # [B, H, R, L]
    d_o = w[..., None] * dout[:, :, None]                                   # [B, H, R, L, D]
    d_lse = w * (np.sum(dout[:, :, None] * o, axis=-1) - np.sum(dout * out, axis=-1)[:, :, None])
    bk = None if buckets is None else np.asarray(buckets)
    dqk = np.zeros((B, H, L, D))
    dv = np.zeros((B, H, L, D))
    for b in range(B):
        for h in range(H):
            x, k_hat, vv = _prep_slice(qk[b, h], v[b, h])
            norms = np.sqrt(np.sum(x * x, axis=1))
            dk_hat = np.zeros((L, D))
            for r in range(n_rounds):
                for k in range(L // chunk):
                    qi, kj, z = _chunk_logits(x, k_hat, perm[b, h, r], k, chunk, self_mask, scale, causal,
                                              None if bk is None else bk[b, h, r], bk[b, h] if union else None)
                    p = np.exp(z - lse[b, h, r, qi][:, None])                   # [c, |W|]
                    g = d_o[b, h, r, qi]                                        # [c, D]
                    dv[b, h, kj] += p.T @ g
                    dz = p * (g @ vv[kj].T - np.sum(g * o[b, h, r, qi], axis=1)[:, None]) \
                        + p * d_lse[b, h, r, qi][:, None]
                    dqk[b, h, qi] += scale * dz @ k_hat[kj]
                    dk_hat[kj] += scale * dz.T @ x[qi]
            small = norms < 1e-12
            proj = np.sum(dk_hat * k_hat, axis=1, keepdims=True) * k_hat
            dqk[b, h] += np.where(small[:, None], dk_hat / 1e-12,
                                  (dk_hat - proj) / np.maximum(norms, 1e-12)[:, None])
    return dqk, dv


def oracle_lsh_attention(qk, v, R, n_buckets: int, chunk: int, self_mask: bool = True,
                         scale: float | None = None, causal: bool = False, bucket_mask: bool = False,
                         union: bool = False):
    """All four steps end to end.  Returns a dict of every intermediate."""
    buckets, near = oracle_hash(qk, R, n_buckets)
    perm = oracle_sort(buckets)
    o, lse = oracle_attend(_f64(qk), _f64(v), perm, chunk, self_mask, scale, causal,
                           buckets if bucket_mask else None, union)
    out, lse_out = oracle_combine(o, lse)
    return {"buckets": buckets, "near_tie": near, "perm": perm, "o_rounds": o,
            "lse_rounds": lse, "out": out, "lse": lse_out}
