"""Approximation error of multi-round LSH attention against full attention, as a
function of the number of hash rounds, on synthetic clustered data (a
training-free analogue of the pages' "more hashes approach full attention";
twgreatdaily ICLR 2020 Reformer article, "1 LSH Attention", multi-round
hashing; nubint.ai review, "제안 방법").

The rows are unit cluster centres plus small noise (the skewed workload's
generator) and the logit scale is large, so each query's attention mass sits
on the keys of its own cluster; the error of the LSH output against dense
self-masked attention over the whole sequence must shrink as rounds are added
(rounds r use the first r projections of one draw, so the key sets are nested).
"""

import math

import numpy as np
import pytest
import torch

import lsh_attention_hash_b200 as lsh
from lsh_attention_hash_b200 import synth
from oracle import oracle_attend, oracle_lsh_attention

ROUNDS = (1, 2, 4, 8)


def _rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.mean(np.linalg.norm(a - b, axis=-1) / np.maximum(np.linalg.norm(b, axis=-1), 1e-30)))


def _clustered(L, D, nb, chunk, n_rounds, seed, dtype="f32"):
    w = synth.small_workload("rounds_err", 1, 1, L, D, dtype, nb, chunk, n_rounds, qk_kind="clusters",
                             n_clusters=16)
    qk, v, R = synth.make_inputs(w, seed=seed)
    return w, qk, v, R


def _assert_shrinks(errs):
    for a, b in zip(errs, errs[1:]):
        assert b <= a * 1.02, errs
    assert errs[-1] < 0.8 * errs[0], errs


def test_oracle_error_against_full_attention_shrinks_with_rounds():
    L, D, nb, chunk, scale = 1024, 32, 32, 32, 8.0
    w, qk, v, R = _clustered(L, D, nb, chunk, max(ROUNDS), seed=3)
    perm_full = np.arange(L, dtype=np.int64)[None, None, None]
    full, _ = oracle_attend(qk.double().numpy(), v.double().numpy(), perm_full, L, True, scale)
    errs = []
    for r in ROUNDS:
        res = oracle_lsh_attention(qk, v, R[:r], nb, chunk, True, scale)
        errs.append(_rel_err(res["out"][0, 0], full[0, 0, 0]))
    _assert_shrinks(errs)


@pytest.mark.gpu
def test_gpu_error_against_full_attention_shrinks_with_rounds():
    """The same study through the C ABI on the 64K workload's shapes at L = 8192 (bf16, D 128,
    chunk 64, 256 buckets): error of the four-call pipeline against dense attention (torch, fp32)."""
    L, D, nb, chunk, scale = 8192, 128, 256, 64, 8.0
    w, qk, v, R = _clustered(L, D, nb, chunk, max(ROUNDS), seed=5, dtype="bf16")
    qk_d, v_d, R_d = qk.cuda(), v.cuda(), R.cuda()
    x = qk_d[0, 0].float()
    kh = x / x.norm(dim=1, keepdim=True).clamp_min(1e-12)
    S = (x @ kh.T) * scale
    S.fill_diagonal_(-math.inf)
    full = torch.softmax(S, dim=1) @ v_d[0, 0].float()
    errs = []
    for r in ROUNDS:
        out = lsh.lsh_attention(qk_d, v_d, R_d[:r].contiguous(), nb, chunk, scale=scale)
        errs.append(_rel_err(out[0, 0].float().cpu(), full.cpu()))
    print("rounds -> mean relative error vs full attention:", dict(zip(ROUNDS, [round(e, 4) for e in errs])))
    _assert_shrinks(errs)
