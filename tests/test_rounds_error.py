"""Approximation quality of multi-round LSH attention against full attention, as a
function of the number of hash rounds, on synthetic clustered data (a
training-free analogue of the pages' "about eight hashes come close to full
attention"; twgreatdaily ICLR 2020 Reformer article, "1 LSH Attention" and
section 4, multi-round hashing; nubint.ai review, "제안 방법").

The rows are unit cluster centres plus small noise (the skewed workload's
generator) and the logit scale is large, so each query's attention mass sits
on the keys of its own cluster.  Rounds r use the first r projections of one
draw, so the rounds' key sets are nested.  Two quantities are reported:

* recall: the share of each query's full-attention softmax mass (dense,
  self-masked, over the whole sequence) that falls on keys inside the union
  of its rounds' chunk windows, averaged over queries.  It can only grow as
  rounds are added (nested unions) and must rise substantially;
* error: the mean distance between the LSH output and the full-attention
  output, divided by the root-mean-square length of the value rows (the
  scale of a typical output), which must shrink.
"""

import math

import numpy as np
import pytest
import torch

import lsh_attention_hash_b200 as lsh
from lsh_attention_hash_b200 import synth
from oracle import oracle_lsh_attention

ROUNDS = (1, 2, 4, 8)


def _clustered(L, D, nb, chunk, n_rounds, seed, dtype="f32"):
    w = synth.small_workload("rounds_err", 1, 1, L, D, dtype, nb, chunk, n_rounds, qk_kind="clusters",
                             n_clusters=16)
    qk, v, R = synth.make_inputs(w, seed=seed)
    return w, qk, v, R


def _window_union(perm_rounds, L, chunk, xp):
    """[L, L] boolean: key j lies in query i's chunk window in some round (self excluded)."""
    M = xp.zeros((L, L), dtype=bool) if xp is np else torch.zeros((L, L), dtype=torch.bool, device="cuda")
    for p in perm_rounds:
        for k in range(L // chunk):
            q = p[k * chunk:(k + 1) * chunk]
            ks = p[max(0, (k - 1) * chunk):(k + 1) * chunk]
            M[q[:, None], ks[None, :]] = True
    idx = xp.arange(L) if xp is np else torch.arange(L, device="cuda")
    M[idx, idx] = False
    return M


def _assert_improves(recalls, errs):
    for a, b in zip(recalls, recalls[1:]):
        assert b >= a - 1e-12, recalls  # nested unions: never less mass
    assert recalls[-1] >= recalls[0] + 0.2, recalls
    for a, b in zip(errs, errs[1:]):
        assert b <= a * 1.02, errs
    assert errs[-1] < 0.7 * errs[0], errs


def test_oracle_recall_and_error_against_full_attention_improve_with_rounds():
    L, D, nb, chunk, scale = 1024, 32, 32, 32, 8.0
    w, qk, v, R = _clustered(L, D, nb, chunk, max(ROUNDS), seed=3)
    x = qk.double().numpy()[0, 0]
    vv = v.double().numpy()[0, 0]
    kh = x / np.maximum(np.linalg.norm(x, axis=1, keepdims=True), 1e-12)
    S = x @ kh.T * scale
    np.fill_diagonal(S, -np.inf)
    W = np.exp(S - S.max(axis=1, keepdims=True))
    W /= W.sum(axis=1, keepdims=True)
    full = W @ vv
    v_rms = math.sqrt(float(np.mean(np.sum(vv * vv, axis=1))))
    recalls, errs = [], []
    for r in ROUNDS:
        res = oracle_lsh_attention(qk, v, R[:r], nb, chunk, True, scale)
        M = _window_union(res["perm"][0, 0], L, chunk, np)
        recalls.append(float((W * M).sum(axis=1).mean()))
        errs.append(float(np.linalg.norm(res["out"][0, 0] - full, axis=1).mean()) / v_rms)
    print("rounds -> recall, error / rms|v|:", dict(zip(ROUNDS, zip(np.round(recalls, 4), np.round(errs, 4)))))
    _assert_improves(recalls, errs)


@pytest.mark.gpu
def test_gpu_recall_and_error_against_full_attention_improve_with_rounds():
    """The same study through the C ABI on the 64K workload's shapes at L = 8192 (bf16, D 128,
    chunk 64, 256 buckets): the four-call pipeline against dense attention (torch, fp32)."""
    L, D, nb, chunk, scale = 8192, 128, 256, 64, 8.0
    w, qk, v, R = _clustered(L, D, nb, chunk, max(ROUNDS), seed=5, dtype="bf16")
    qk_d, v_d, R_d = qk.cuda(), v.cuda(), R.cuda()
    x = qk_d[0, 0].float()
    kh = x / x.norm(dim=1, keepdim=True).clamp_min(1e-12)
    S = (x @ kh.T) * scale
    S.fill_diagonal_(-math.inf)
    W = torch.softmax(S, dim=1)
    vv = v_d[0, 0].float()
    full = W @ vv
    v_rms = float(vv.pow(2).sum(dim=1).mean().sqrt())
    recalls, errs = [], []
    for r in ROUNDS:
        res = lsh.lsh_attention(qk_d, v_d, R_d[:r].contiguous(), nb, chunk, scale=scale, return_all=True)
        M = _window_union(res["perm"][0, 0].long(), L, chunk, torch)
        recalls.append(float((W * M).sum(dim=1).mean()))
        errs.append(float((res["out"][0, 0].float() - full).norm(dim=1).mean()) / v_rms)
    print("rounds -> recall, error / rms|v|:", dict(zip(ROUNDS, zip([round(a, 4) for a in recalls],
                                                                    [round(e, 4) for e in errs]))))
    _assert_improves(recalls, errs)
