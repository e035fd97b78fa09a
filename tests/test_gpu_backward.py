"""Parity of the backward (lsh_chunk_attend_backward, through the C ABI) with the float64 oracle.

The forward runs through the four calls (its merged output and LSE feed the
backward); the oracle recomputes everything from the same inputs, the GPU's
perm and buckets.  Tolerance on dqk and dv: max-abs error <= tol * max(1,
max |reference|), tol 1e-4 when the forward's output is fp32 and 2e-2 when it
is bf16 (the backward reads the stored output in dout . out).
"""

import zlib

import numpy as np
import pytest
import torch

import lsh_attention_hash_b200 as lsh
from lsh_attention_hash_b200 import synth
from oracle import oracle_attend_backward
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def _run(w, seed, self_mask=True, causal=False, bucket_mask=False, union=False, scale=None):
    qk, v, R = synth.make_inputs(w, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(qk.shape, generator=g).to(w.torch_dtype)
    qk_d, v_d, R_d, dout_d = qk.to(DEV), v.to(DEV), R.to(DEV), dout.to(DEV)
    res = lsh.lsh_attention(qk_d, v_d, R_d, w.n_buckets, w.chunk, self_mask=self_mask, causal=causal,
                            bucket_mask=bucket_mask, union=union, scale=scale, return_all=True)
    dqk, dv = lsh.lsh_chunk_attend_backward(qk_d, v_d, res["perm"], w.chunk, res["out"], res["lse"], dout_d,
                                            self_mask=self_mask, causal=causal, buckets=res["buckets"],
                                            bucket_mask=bucket_mask, union=union, scale=scale)
    torch.cuda.synchronize()
    assert lsh.lsh_get_device_status() == 0
    return qk, v, dout, res, dqk, dv


def _check(qk, v, dout, res, dqk, dv, chunk, dtype, slices=None, **kw):
    perm = parity.np_(res["perm"])
    bk = parity.np_(res["buckets"]) if kw.get("bucket_mask") else None
    sel = slices or [(b, h) for b in range(qk.shape[0]) for h in range(qk.shape[1])]
    worst = 0.0
    for (b, h) in sel:
        rq, rv = oracle_attend_backward(
            parity.f64(qk[b, h])[None, None], parity.f64(v[b, h])[None, None], perm[b, h][None, None], chunk,
            parity.f64(dout[b, h])[None, None], kw.get("self_mask", True), kw.get("scale"),
            kw.get("causal", False), None if bk is None else bk[b, h][None, None], kw.get("union", False))
        for ref, got, name in ((rq[0, 0], dqk[b, h], "dqk"), (rv[0, 0], dv[b, h], "dv")):
            err = float(np.max(np.abs(ref - parity.f64(got))))
            bound = TOL[dtype] * max(1.0, float(np.max(np.abs(ref))))
            assert err <= bound, f"{name} slice {(b, h)}: max-abs error {err:.3e} > {bound:.3e}"
            worst = max(worst, err / bound)
    return worst


@pytest.mark.parametrize("name,shape,kw", [
    ("bwd_tiny", (1, 1, 64, 32, "f32", 8, 8, 2), dict()),
    ("bwd_causal", (1, 2, 256, 32, "f32", 16, 16, 3), dict(causal=True)),
    ("bwd_tc_fwd", (2, 2, 1024, 128, "bf16", 16, 64, 2), dict()),        # forward on the tensor cores
    ("bwd_bucket_tc_fwd", (1, 2, 1024, 64, "bf16", 32, 64, 2), dict(bucket_mask=True)),
    ("bwd_bucket_union", (1, 2, 512, 64, "f32", 8, 32, 4), dict(bucket_mask=True, union=True)),
    ("bwd_chunk1", (1, 1, 64, 32, "f32", 8, 1, 2), dict()),             # chunk 0 sees only itself
    ("bwd_union_causal", (1, 3, 320, 64, "bf16", 8, 32, 3), dict(bucket_mask=True, union=True, causal=True)),
    ("bwd_dense", (1, 1, 256, 64, "f32", 16, 256, 2), dict()),          # chunk = L
    ("bwd_d256", (1, 1, 256, 256, "f32", 8, 32, 2), dict(scale=0.2)),
    ("bwd_noself", (1, 2, 256, 64, "f32", 16, 32, 2), dict(self_mask=False, bucket_mask=True)),
])
def test_backward_matches_oracle(name, shape, kw):
    w = synth.small_workload(name, *shape)
    qk, v, dout, res, dqk, dv = _run(w, zlib.crc32(name.encode()) % 1000, **kw)
    _check(qk, v, dout, res, dqk, dv, w.chunk, w.torch_dtype, **kw)


def test_backward_is_deterministic():
    w = synth.small_workload("bwd_det", 1, 2, 1024, 64, "bf16", 32, 64, 2)
    qk, v, dout, res, dqk, dv = _run(w, 3, bucket_mask=True)
    dqk2, dv2 = lsh.lsh_chunk_attend_backward(qk.to(DEV), v.to(DEV), res["perm"], w.chunk, res["out"], res["lse"],
                                              dout.to(DEV), buckets=res["buckets"], bucket_mask=True)
    torch.cuda.synchronize()
    assert torch.equal(dqk, dqk2) and torch.equal(dv, dv2)


# The tensor-core backward serves bf16, D 128, chunk 64, L % 128 == 0 and every mask (the union
# correction up to 8 rounds): work units of 16 fills (2048 tokens), so L > 2048 has leading and half
# fills between units.
@pytest.mark.parametrize("name,shape,kw", [
    ("bwd_tc_one_fill", (1, 1, 128, 128, "bf16", 16, 64, 1), dict()),
    ("bwd_tc_units", (1, 2, 4096, 128, "bf16", 64, 64, 2), dict()),
    ("bwd_tc_ragged_units_noself", (1, 1, 5120, 128, "bf16", 64, 64, 3), dict(self_mask=False)),
    ("bwd_tc_scale", (2, 1, 1024, 128, "bf16", 32, 64, 2), dict(scale=0.5)),
])
def test_tensor_core_backward_matches_oracle(name, shape, kw):
    w = synth.small_workload(name, *shape)
    qk, v, dout, res, dqk, dv = _run(w, zlib.crc32(name.encode()) % 1000, **kw)
    _check(qk, v, dout, res, dqk, dv, w.chunk, w.torch_dtype, **kw)


# The masks on the tensor-core backward: positions, buckets and (union) every round's bucket land with
# each row; queries that their masks leave alone keep their own key.
@pytest.mark.parametrize("name,shape,kw", [
    ("bwd_tc_causal", (1, 2, 1024, 128, "bf16", 16, 64, 2), dict(causal=True)),
    ("bwd_tc_bucket", (1, 2, 1024, 128, "bf16", 32, 64, 2), dict(bucket_mask=True)),
    ("bwd_tc_bucket_union", (1, 2, 1024, 128, "bf16", 16, 64, 3), dict(bucket_mask=True, union=True)),
    ("bwd_tc_causal_bucket_union", (1, 1, 4096, 128, "bf16", 64, 64, 4),
     dict(causal=True, bucket_mask=True, union=True)),
    ("bwd_tc_causal_bucket_noself", (1, 1, 2560, 128, "bf16", 32, 64, 2),
     dict(causal=True, bucket_mask=True, self_mask=False)),
])
def test_tensor_core_backward_masks_match_oracle(name, shape, kw):
    w = synth.small_workload(name, *shape)
    qk, v, dout, res, dqk, dv = _run(w, zlib.crc32(name.encode()) % 1000, **kw)
    _check(qk, v, dout, res, dqk, dv, w.chunk, w.torch_dtype, **kw)


@pytest.mark.parametrize("kw", [dict(), dict(causal=True), dict(bucket_mask=True, union=True)],
                         ids=["plain", "causal", "bucket_union"])
def test_tensor_core_backward_more_units_than_sms(kw):
    """160 one-fill units: every persistent CTA walks several (b, h) slices, with each mask's per-row
    tables landing in slots that earlier units used."""
    w = synth.small_workload("bwd_tc_many", 10, 16, 128, 128, "bf16", 16, 64, 2)
    qk, v, dout, res, dqk, dv = _run(w, 11, **kw)
    _check(qk, v, dout, res, dqk, dv, w.chunk, w.torch_dtype, slices=[(0, 0), (3, 7), (9, 15), (5, 0)], **kw)


@pytest.mark.parametrize("kw", [dict(), dict(causal=True, bucket_mask=True, union=True)], ids=["plain", "all_masks"])
def test_tensor_core_backward_is_deterministic(kw):
    w = synth.small_workload("bwd_tc_det", 1, 2, 4096, 128, "bf16", 64, 64, 2)
    qk, v, dout, res, dqk, dv = _run(w, 5, **kw)
    dqk2, dv2 = lsh.lsh_chunk_attend_backward(qk.to(DEV), v.to(DEV), res["perm"], w.chunk, res["out"], res["lse"],
                                              dout.to(DEV), buckets=res["buckets"] if kw else None, **kw)
    torch.cuda.synchronize()
    assert torch.equal(dqk, dqk2) and torch.equal(dv, dv2)


@pytest.mark.slow
def test_64k_workload_backward_one_slice():
    """The full-size backward launch (B 8, H 8, L 65536, D 128, bf16, 1024 buckets, chunk 64, 8 rounds),
    slice (3, 5) checked in full against the oracle."""
    w = synth.WORKLOADS["64k"]
    qk, v, dout, res, dqk, dv = _run(w, 0)
    _check(qk, v, dout, res, dqk, dv, w.chunk, w.torch_dtype, slices=[(3, 5)])
