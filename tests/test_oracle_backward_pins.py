"""Pins of the float64 backward oracle (CPU only).

The backward differentiates sum(dout * out) through the round merge and each
round's chunk attention with the hash, the sort and the masks held fixed.  It
is pinned by central finite differences of the forward oracle (a different
route: no chain rule at all), by torch autograd of dense attention with
normalised keys at c = L (a library routine on the plain formula), and by two
invariants of the method: the merged weights of a query sum to one, so the
value gradients add up to the output gradients, and the output is linear in
the values, so the value gradient does not depend on them.
"""

import math
import zlib

import numpy as np
import pytest
import torch

from oracle import oracle_attend, oracle_attend_backward, oracle_combine


def _loss(qk, v, perm, chunk, dout, **kw):
    o, lse = oracle_attend(qk, v, perm, chunk, **kw)
    out, _ = oracle_combine(o, lse)
    return float(np.sum(out * dout))


def _finite_diff(qk, v, perm, chunk, dout, eps=1e-6, **kw):
    gq = np.zeros_like(qk)
    gv = np.zeros_like(v)
    for a, g in ((qk, gq), (v, gv)):
        for idx in np.ndindex(a.shape):
            old = a[idx]
            a[idx] = old + eps
            up = _loss(qk, v, perm, chunk, dout, **kw)
            a[idx] = old - eps
            dn = _loss(qk, v, perm, chunk, dout, **kw)
            a[idx] = old
            g[idx] = (up - dn) / (2 * eps)
    return gq, gv


def _case(seed, L, D, nr, nb, sorted_perm=True):
    rng = np.random.default_rng(seed)
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    dout = rng.standard_normal((1, 1, L, D))
    bk = rng.integers(0, nb, size=(nr, L)).astype(np.int32)
    if sorted_perm:
        perm = np.stack([np.argsort(bk[r], kind="stable") for r in range(nr)]).astype(np.int32)
    else:
        perm = np.stack([rng.permutation(L) for _ in range(nr)]).astype(np.int32)
    return qk, v, dout, bk[None, None], perm[None, None]


@pytest.mark.parametrize("name,L,chunk,kw", [
    ("plain", 12, 4, dict(self_mask=True, scale=0.9)),
    ("no_self_mask", 12, 4, dict(self_mask=False, scale=1.3)),
    ("chunk1", 8, 1, dict(self_mask=True, scale=0.7)),          # chunk 0 sees only itself
    ("single_chunk", 10, 10, dict(self_mask=True, scale=0.8)),
    ("causal", 12, 3, dict(self_mask=True, scale=1.1, causal=True)),
    ("bucket", 12, 4, dict(self_mask=True, scale=0.9, bucket=True)),
    ("bucket_union", 12, 4, dict(self_mask=True, scale=1.2, bucket=True, union=True)),
    ("bucket_union_causal", 12, 6, dict(self_mask=True, scale=1.0, bucket=True, union=True, causal=True)),
])
def test_backward_matches_central_finite_differences(name, L, chunk, kw):
    kw = dict(kw)
    D, nr, nb = 3, 3, 3
    qk, v, dout, bk, perm = _case(zlib.crc32(name.encode()) % 1000, L, D, nr, nb, sorted_perm=name != "plain")
    if kw.pop("bucket", False):
        kw["buckets"] = bk
    gq, gv = oracle_attend_backward(qk, v, perm, chunk, dout, **kw)
    fq, fv = _finite_diff(qk.copy(), v.copy(), perm, chunk, dout, **kw)
    scale_q = max(1.0, float(np.max(np.abs(fq))))
    assert np.max(np.abs(gq - fq)) < 1e-7 * scale_q, (np.max(np.abs(gq - fq)), scale_q)
    assert np.max(np.abs(gv - fv)) < 1e-7 * max(1.0, float(np.max(np.abs(fv))))


@pytest.mark.parametrize("self_mask", [False, True])
def test_backward_single_chunk_matches_autograd_of_dense_attention(self_mask):
    """c = L, one round: dense softmax attention with normalised keys, differentiated by torch autograd."""
    rng = np.random.default_rng(5)
    L, D, scale = 16, 6, 0.6
    qk = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    dout = rng.standard_normal((1, 1, L, D))
    perm = rng.permutation(L).astype(np.int32)[None, None, None]
    gq, gv = oracle_attend_backward(qk, v, perm, L, dout, self_mask=self_mask, scale=scale)
    x = torch.tensor(qk[0, 0], requires_grad=True)
    vt = torch.tensor(v[0, 0], requires_grad=True)
    k = x / x.norm(dim=1, keepdim=True)
    s = scale * x @ k.T
    if self_mask:
        s = s.masked_fill(torch.eye(L, dtype=torch.bool), float("-inf"))
    out = torch.softmax(s, dim=1) @ vt
    (out * torch.tensor(dout[0, 0])).sum().backward()
    assert np.allclose(gq[0, 0], x.grad.numpy(), atol=1e-12)
    assert np.allclose(gv[0, 0], vt.grad.numpy(), atol=1e-12)


@pytest.mark.parametrize("kw", [dict(), dict(causal=True), dict(bucket=True), dict(bucket=True, union=True)])
def test_backward_value_gradients_sum_to_output_gradients_and_ignore_values(kw):
    kw = dict(kw)
    rng = np.random.default_rng(17)
    L, D, nr, chunk = 32, 4, 4, 8
    qk, v, dout, bk, perm = _case(17, L, D, nr, 4)
    if kw.pop("bucket", False):
        kw["buckets"] = bk
    gq, gv = oracle_attend_backward(qk, v, perm, chunk, dout, **kw)
    assert np.allclose(gv.sum(axis=2), dout.sum(axis=2), atol=1e-12)
    v2 = v + rng.standard_normal(v.shape)
    gq2, gv2 = oracle_attend_backward(qk, 3.0 * v2, perm, chunk, dout, **kw)
    assert np.allclose(gv2, gv, atol=1e-12)
    gq3, _ = oracle_attend_backward(qk, 3.0 * v, perm, chunk, dout, **kw)
    assert np.allclose(gq3, 3.0 * gq, atol=1e-10)


def test_backward_default_scale_is_inverse_sqrt_d():
    qk, v, dout, _, perm = _case(23, 16, 4, 2, 4)
    a = oracle_attend_backward(qk, v, perm, 4, dout)
    b = oracle_attend_backward(qk, v, perm, 4, dout, scale=1 / math.sqrt(4))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
