"""Parity of the CUDA path (called through the C ABI) with the float64 oracle.

Every test here needs a B200.  Inputs come from lsh_attention_hash_b200.synth;
expected values come only from oracle/.  See tests/parity.py for the rules
(bit-exact buckets except near ties, bit-exact perm, max-abs tolerance on
outputs: 1e-4 for fp32 inputs, 2e-2 for bf16 inputs).
"""

import zlib

import numpy as np
import pytest
import torch

import lsh_attention_hash_b200 as lsh
from lsh_attention_hash_b200 import synth
from oracle import oracle_combine, oracle_hash, oracle_sort
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_gpu(w, qk, v, R, self_mask=True, scale=None, out_dtype=None, **masks):
    qk_d, v_d, R_d = qk.to(DEV), v.to(DEV), R.to(DEV)
    res = lsh.lsh_attention(qk_d, v_d, R_d, w.n_buckets, w.chunk, self_mask=self_mask, scale=scale,
                            return_all=True, **masks)
    torch.cuda.synchronize()
    assert lsh.lsh_get_device_status() == 0
    return res


def full_parity(w, qk, v, R, self_mask=True, scale=None, max_flag_frac=1e-3):
    res = run_gpu(w, qk, v, R, self_mask, scale)
    mism, flagged = parity.check_hash(qk, R, w.n_buckets, res["buckets"], res["near_tie"], max_flag_frac)
    parity.check_sort(res["buckets"], res["perm"])
    parity.check_attend(qk, v, res["perm"], w.chunk, self_mask, scale, res["o_rounds"], res["lse_rounds"],
                        w.torch_dtype)
    parity.check_combine(res["o_rounds"], res["lse_rounds"], res["out"], res["lse"], w.torch_dtype)
    if mism == 0:  # all buckets agree: the whole pipeline must agree with the oracle's own run
        from oracle import oracle_lsh_attention

        ref = oracle_lsh_attention(qk, v, R, w.n_buckets, w.chunk, self_mask, scale)
        assert np.array_equal(ref["perm"], parity.np_(res["perm"]))
        err = float(np.max(np.abs(ref["out"] - parity.f64(res["out"]))))
        assert err <= parity.TOL[w.torch_dtype], err
    return res, mism, flagged


def test_tiny_workload_end_to_end():
    w = synth.WORKLOADS["tiny"]
    qk, v, R = synth.make_inputs(w)
    _, mism, _ = full_parity(w, qk, v, R)
    assert mism == 0


def test_4k_workload_end_to_end():
    w = synth.WORKLOADS["4k"]
    qk, v, R = synth.make_inputs(w)
    full_parity(w, qk, v, R)


EDGE_CASES = [
    # name, B, H, L, D, dtype, n_buckets, chunk, n_rounds, self_mask
    ("ragged_rows_bf16", 1, 3, 200, 64, "bf16", 16, 8, 3, True),
    ("chunk1_self_only", 1, 2, 64, 64, "bf16", 8, 1, 2, True),
    ("chunk_eq_L", 2, 1, 256, 128, "bf16", 32, 256, 2, True),
    ("two_chunks", 1, 2, 128, 128, "bf16", 8, 64, 2, True),
    ("no_self_mask", 2, 2, 512, 128, "bf16", 16, 64, 2, False),
    ("two_buckets", 1, 2, 384, 64, "bf16", 2, 64, 3, True),
    ("fp32_odd_sizes", 1, 3, 120, 40, "f32", 10, 12, 2, True),
    ("fp32_d256", 1, 1, 256, 256, "f32", 64, 32, 1, True),
    ("many_buckets", 1, 1, 2048, 64, "bf16", 4096, 64, 2, True),
    ("big_chunk", 1, 1, 4096, 64, "bf16", 8, 2048, 1, True),
    # chunk 64 bf16 (tensor-core kernel): odd chunk count, one chunk, several work units per segment
    ("tc_odd_chunks", 1, 2, 192, 128, "bf16", 8, 64, 2, True),
    ("tc_single_chunk", 2, 1, 64, 64, "bf16", 4, 64, 3, True),
    ("tc_units_d64", 1, 1, 8256, 64, "bf16", 128, 64, 2, True),
    ("tc_units_d128_nomask", 1, 2, 8192, 128, "bf16", 128, 64, 1, False),
    # shapes served by the tensor-core hash: ragged 128-row tiles, 1..4 column chunks per round
    ("tc_hash_d64_nb2048", 1, 2, 1000, 64, "bf16", 2048, 8, 2, True),
    ("tc_hash_d128_nb128_ragged", 2, 3, 200, 128, "bf16", 128, 8, 3, True),
    ("tc_hash_d128_nb1024", 1, 1, 4096, 128, "bf16", 1024, 64, 2, True),
    ("tc_hash_d64_nb512_many_rounds", 1, 1, 1024, 64, "bf16", 512, 64, 9, True),
]


@pytest.mark.parametrize("case", EDGE_CASES, ids=[c[0] for c in EDGE_CASES])
def test_edge_cases(case):
    name, B, H, L, D, dt, nb, c, nr, sm = case
    w = synth.small_workload(name, B, H, L, D, dt, nb, c, nr)
    qk, v, R = synth.make_inputs(w, seed=zlib.crc32(name.encode()) % 1000)
    full_parity(w, qk, v, R, self_mask=sm)


def test_zero_rows_and_custom_scale():
    w = synth.small_workload("zero", 1, 1, 256, 64, "bf16", 16, 32, 2)
    qk, v, R = synth.make_inputs(w, seed=3)
    qk[0, 0, 5] = 0
    qk[0, 0, 77] = 0
    res = run_gpu(w, qk, v, R, scale=0.3)
    nb = res["buckets"].cpu()
    assert nb[0, 0, :, 5].tolist() == [0, 0] and nb[0, 0, :, 77].tolist() == [0, 0]
    assert res["near_tie"].cpu()[0, 0, :, 5].tolist() == [1, 1]
    # the two planted zero rows are near ties in both rounds: 4 of 512 hashes
    full_parity(w, qk, v, R, scale=0.3, max_flag_frac=4 / 512 + 1e-3)


@pytest.mark.parametrize("nb", [16, 256])
def test_zero_rows_get_bucket_zero(nb):
    """A zero row has p = 0 everywhere: bucket 0 (first maximum), flagged as a near tie."""
    w = synth.small_workload("zero_nb", 1, 2, 256, 128, "bf16", nb, 64, 2)
    qk, v, R = synth.make_inputs(w, seed=8)
    qk[0, 1, 0] = 0
    qk[0, 0, 131] = 0
    b, f = lsh.lsh_hash(qk.to(DEV), R.to(DEV), nb)
    b, f = b.cpu(), f.cpu()
    assert b[0, 1, :, 0].tolist() == [0, 0] and b[0, 0, :, 131].tolist() == [0, 0]
    assert f[0, 1, :, 0].tolist() == [1, 1] and f[0, 0, :, 131].tolist() == [1, 1]


def test_hash_with_and_without_flags_agree():
    """The near-tie output is optional; the buckets must not depend on asking for it."""
    for nb in (32, 256, 1024):
        w = synth.small_workload("flags", 2, 2, 1536, 128, "bf16", nb, 64, 3)
        qk, v, R = synth.make_inputs(w, seed=nb)
        b1, f1 = lsh.lsh_hash(qk.to(DEV), R.to(DEV), nb)
        b2, f2 = lsh.lsh_hash(qk.to(DEV), R.to(DEV), nb, with_near_tie=False)
        assert f2 is None and torch.equal(b1, b2)


@pytest.mark.parametrize("scale", [0.02, 6.0, 40.0])
def test_chunk64_attention_scales(scale):
    """Small and large logit scales on the tensor-core attention (40: the row sums underflow
    under the Cauchy-Schwarz shift, so the kernel falls back to the exact maximum)."""
    w = synth.small_workload("scales", 1, 2, 1024, 128, "bf16", 16, 64, 2)
    qk, v, R = synth.make_inputs(w, seed=9)
    full_parity(w, qk, v, R, scale=scale)


def test_fp32_output_from_bf16_input():
    w = synth.small_workload("f32out", 2, 2, 512, 128, "bf16", 16, 64, 2)
    qk, v, R = synth.make_inputs(w, seed=4)
    qk_d, v_d, R_d = qk.to(DEV), v.to(DEV), R.to(DEV)
    b, _ = lsh.lsh_hash(qk_d, R_d, w.n_buckets)
    perm, _, _, _ = lsh.lsh_sort_permute(b, w.n_buckets)
    o, lse = lsh.lsh_chunk_attend(qk_d, v_d, perm, w.chunk, out_dtype=torch.float32)
    out, lse_out = lsh.lsh_combine_rounds(o, lse, out_dtype=torch.float32)
    torch.cuda.synchronize()
    parity.check_attend(qk, v, perm, w.chunk, True, None, o, lse, torch.bfloat16)
    ref, _ = oracle_combine(parity.f64(o), parity.f64(lse))
    assert np.max(np.abs(ref - parity.f64(out))) < 1e-5  # fp32 in, fp32 out


def test_sorted_gather_and_inverse():
    w = synth.small_workload("gather", 2, 2, 1024, 128, "bf16", 32, 64, 3)
    qk, v, R = synth.make_inputs(w, seed=5)
    qk_d, v_d, R_d = qk.to(DEV), v.to(DEV), R.to(DEV)
    b, _ = lsh.lsh_hash(qk_d, R_d, w.n_buckets)
    perm, inv, qs, vs = lsh.lsh_sort_permute(b, w.n_buckets, want_inv=True, qk=qk_d, v=v_d)
    o1, l1 = lsh.lsh_chunk_attend(qk_d, v_d, perm, w.chunk)
    o2, l2 = lsh.lsh_chunk_attend(qk_d, v_d, perm, w.chunk, qk_sorted=qs, v_sorted=vs)
    torch.cuda.synchronize()
    p = perm.long()
    idx = torch.arange(w.L, device=DEV).expand_as(p)
    assert torch.equal(torch.gather(inv.long(), -1, p), idx)
    for r in range(w.n_rounds):
        assert torch.equal(qs[:, :, r], torch.gather(qk_d, 2, p[:, :, r, :, None].expand(-1, -1, -1, w.D)))
        assert torch.equal(vs[:, :, r], torch.gather(v_d, 2, p[:, :, r, :, None].expand(-1, -1, -1, w.D)))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_deterministic_reruns():
    w = synth.small_workload("det", 2, 2, 2048, 128, "bf16", 64, 64, 2)
    qk, v, R = synth.make_inputs(w, seed=6)
    a = run_gpu(w, qk, v, R)
    b = run_gpu(w, qk, v, R)
    for k in ("buckets", "near_tie", "perm", "o_rounds", "lse_rounds", "out", "lse"):
        assert torch.equal(a[k], b[k]), k


def test_out_of_range_bucket_is_recorded_not_faulted():
    """A host-made failure: bucket ids outside [0, n_buckets) are skipped and reported."""
    buckets = torch.zeros((1, 1, 1, 1024), dtype=torch.int32, device=DEV)
    buckets[0, 0, 0, 10] = 99
    buckets[0, 0, 0, 11] = -3
    perm = torch.full_like(buckets, -1)
    lsh.lsh_sort_permute(buckets, 16, perm=perm)
    assert lsh.lsh_get_device_status() == 1  # LSH_ERR_INVALID_ARG
    assert lsh.lsh_get_device_status() == 0  # cleared by the read
    p = perm.cpu()[0, 0, 0]
    assert p[:1022].tolist() == [i for i in range(1024) if i not in (10, 11)]


def _sampled_slices(w, slices, row_sample=None, slot_sample=None, bucket_mask=False, union=False):
    qk, v, R = synth.make_inputs(w)
    res = run_gpu(w, qk, v, R, bucket_mask=bucket_mask, union=union)
    for (b, h) in slices:
        qk_bh, v_bh = qk[b, h], v[b, h]
        rows = np.arange(w.L) if row_sample is None else np.sort(
            np.random.default_rng(b * 100 + h).choice(w.L, row_sample, replace=False))
        g_b = res["buckets"][b, h].cpu()
        g_f = res["near_tie"][b, h].cpu()
        parity.check_hash(qk_bh[rows][None, None], R, w.n_buckets, g_b[:, rows][None, None],
                          g_f[:, rows][None, None])
        parity.check_sort(g_b[None, None], res["perm"][b, h].cpu()[None, None])
        slots = None if slot_sample is None else np.sort(
            np.random.default_rng(b * 7 + h).choice(w.L, slot_sample, replace=False))
        parity.check_slice_rounds(qk_bh, v_bh, res["perm"][b, h].cpu(), w.chunk, True, None,
                                  res["o_rounds"][b, h].cpu(), res["lse_rounds"][b, h].cpu(), w.torch_dtype,
                                  slots, g_b if bucket_mask else None, union)
        parity.check_combine(res["o_rounds"][b, h][None, None], res["lse_rounds"][b, h][None, None],
                             res["out"][b, h][None, None], res["lse"][b, h][None, None], w.torch_dtype)
    return res


def test_skewed_workload_sampled_slices():
    w = synth.WORKLOADS["skewed16k"]
    res = _sampled_slices(w, [(0, 0), (5, 3)])
    # the workload is meant to be uneven: the largest bucket is many times the mean
    counts = torch.bincount(res["buckets"][0, 0, 0].long(), minlength=w.n_buckets)
    assert counts.max().item() > 8 * w.L / w.n_buckets


@pytest.mark.slow
def test_64k_workload_sampled_slices():
    w = synth.WORKLOADS["64k"]
    _sampled_slices(w, [(0, 0), (7, 7)], slot_sample=4096)


@pytest.mark.slow
def test_1m_workload_sampled_slices():
    w = synth.WORKLOADS["1m"]
    _sampled_slices(w, [(0, 0), (0, 6)], row_sample=4096, slot_sample=2048)


# ---------------------------------------------------------------- causal variant
@pytest.mark.parametrize("name,shape", [
    ("causal_tiny", (1, 1, 1024, 64, "f32", 16, 64, 1)),
    ("causal_bf16", (2, 2, 2048, 128, "bf16", 32, 64, 2)),
    ("causal_dense", (1, 2, 256, 128, "bf16", 16, 256, 2)),    # chunk = L: dense causal attention
    ("causal_chunk1", (1, 1, 64, 32, "f32", 8, 1, 1)),          # every window has two slots
    ("causal_ragged", (1, 3, 320, 64, "bf16", 8, 32, 3)),
    ("causal_tc_d64_odd", (1, 2, 8256, 64, "bf16", 128, 64, 2)),   # tensor-core path, odd chunk count
])
def test_causal_attention_end_to_end(name, shape):
    """Keys after the query's original position are not admissible; a query with no earlier key in
    its window sees only itself.  Checked stage by stage and end to end against the oracle."""
    w = synth.small_workload(name, *shape)
    qk, v, R = synth.make_inputs(w, seed=zlib.crc32(name.encode()) % 1000)
    qk_d, v_d, R_d = qk.to(DEV), v.to(DEV), R.to(DEV)
    res = lsh.lsh_attention(qk_d, v_d, R_d, w.n_buckets, w.chunk, causal=True, return_all=True)
    torch.cuda.synchronize()
    assert lsh.lsh_get_device_status() == 0
    mism, _ = parity.check_hash(qk, R, w.n_buckets, res["buckets"], res["near_tie"], 1e-3)
    parity.check_sort(res["buckets"], res["perm"])
    parity.check_attend(qk, v, res["perm"], w.chunk, True, None, res["o_rounds"], res["lse_rounds"],
                        w.torch_dtype, causal=True)
    parity.check_combine(res["o_rounds"], res["lse_rounds"], res["out"], res["lse"], w.torch_dtype)
    if mism == 0:
        from oracle import oracle_lsh_attention

        ref = oracle_lsh_attention(qk, v, R, w.n_buckets, w.chunk, causal=True)
        err = float(np.max(np.abs(ref["out"] - parity.f64(res["out"]))))
        assert err <= parity.TOL[w.torch_dtype], err


@pytest.mark.parametrize("scale", [None, 6.0, 40.0])
def test_causal_tensor_core_attention_scales(scale):
    """The tensor-core attention with the causal mask (bf16, chunk 64): rows with no earlier key see
    only themselves; at scale 40 the Cauchy-Schwarz shift underflows and the exact-maximum path
    (with the causal mask) takes over."""
    w = synth.small_workload("causal_tc", 2, 2, 4096, 128, "bf16", 64, 64, 2)
    qk, v, R = synth.make_inputs(w, seed=31)
    qk_d, v_d, R_d = qk.to(DEV), v.to(DEV), R.to(DEV)
    b, _ = lsh.lsh_hash(qk_d, R_d, w.n_buckets)
    perm, _, _, _ = lsh.lsh_sort_permute(b, w.n_buckets)
    o, l = lsh.lsh_chunk_attend(qk_d, v_d, perm, w.chunk, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert lsh.lsh_get_device_status() == 0
    parity.check_attend(qk, v, perm, w.chunk, True, scale, o, l, w.torch_dtype, causal=True)


# ------------------------------------------------- bucket-equality mask and union
@pytest.mark.parametrize("name,shape,causal,union", [
    ("bucket_tiny", (1, 1, 64, 32, "f32", 8, 8, 2), False, False),
    ("bucket_union_f32", (1, 2, 512, 64, "f32", 4, 32, 8), False, True),     # few buckets: many shared rounds
    ("bucket_union_bf16", (2, 2, 2048, 128, "bf16", 32, 64, 4), False, True),
    ("bucket_dense", (1, 2, 256, 64, "bf16", 16, 256, 2), False, False),     # chunk = L
    ("bucket_chunk1", (1, 1, 64, 32, "f32", 8, 1, 2), False, True),          # every window has two slots
    ("bucket_union_causal", (1, 3, 320, 64, "bf16", 8, 32, 3), True, True),
    ("bucket_many", (1, 1, 4096, 128, "bf16", 1024, 64, 2), False, True),    # most buckets split or alone
    # tensor-core path (bf16, chunk 64, D 64 / 128, no union)
    ("bucket_tc", (2, 2, 4096, 128, "bf16", 64, 64, 2), False, False),
    ("bucket_tc_many", (1, 2, 4096, 128, "bf16", 1024, 64, 2), False, False),  # many rows alone
    ("bucket_tc_causal_d64_odd", (1, 2, 8256, 64, "bf16", 128, 64, 2), True, False),
    ("bucket_tc_3heads", (1, 3, 2048, 64, "bf16", 32, 64, 3), False, False),
])
def test_bucket_mask_attention_end_to_end(name, shape, causal, union):
    """Keys outside the query's bucket are not admissible (a query alone in its bucket sees only
    itself); with the union correction each logit is lowered by log(#rounds sharing the bucket).
    Checked stage by stage and end to end against the oracle."""
    w = synth.small_workload(name, *shape)
    qk, v, R = synth.make_inputs(w, seed=zlib.crc32(name.encode()) % 1000)
    qk_d, v_d, R_d = qk.to(DEV), v.to(DEV), R.to(DEV)
    res = lsh.lsh_attention(qk_d, v_d, R_d, w.n_buckets, w.chunk, causal=causal, bucket_mask=True, union=union,
                            return_all=True)
    torch.cuda.synchronize()
    assert lsh.lsh_get_device_status() == 0
    mism, _ = parity.check_hash(qk, R, w.n_buckets, res["buckets"], res["near_tie"], 1e-3)
    parity.check_sort(res["buckets"], res["perm"])
    parity.check_attend(qk, v, res["perm"], w.chunk, True, None, res["o_rounds"], res["lse_rounds"],
                        w.torch_dtype, causal=causal, g_buckets=res["buckets"], union=union)
    parity.check_combine(res["o_rounds"], res["lse_rounds"], res["out"], res["lse"], w.torch_dtype)
    if mism == 0:
        from oracle import oracle_lsh_attention

        ref = oracle_lsh_attention(qk, v, R, w.n_buckets, w.chunk, causal=causal, bucket_mask=True, union=union)
        err = float(np.max(np.abs(ref["out"] - parity.f64(res["out"]))))
        assert err <= parity.TOL[w.torch_dtype], err


def test_bucket_mask_without_self_mask_and_custom_scale():
    """self_mask off: a query always sees itself (it shares its own bucket); scale 3."""
    w = synth.small_workload("bucket_noself", 1, 2, 1024, 64, "f32", 16, 32, 3)
    qk, v, R = synth.make_inputs(w, seed=5)
    qk_d, v_d, R_d = qk.to(DEV), v.to(DEV), R.to(DEV)
    b, _ = lsh.lsh_hash(qk_d, R_d, w.n_buckets)
    perm, _, _, _ = lsh.lsh_sort_permute(b, w.n_buckets)
    o, l = lsh.lsh_chunk_attend(qk_d, v_d, perm, w.chunk, self_mask=False, buckets=b, bucket_mask=True,
                                union=True, scale=3.0)
    torch.cuda.synchronize()
    assert lsh.lsh_get_device_status() == 0
    parity.check_attend(qk, v, perm, w.chunk, False, 3.0, o, l, w.torch_dtype, g_buckets=b, union=True)


@pytest.mark.slow
def test_64k_workload_bucket_union_sampled_slices():
    """The full-size launch (B 8, H 8, L 65536, D 128, bf16, 1024 buckets, chunk 64, 8 rounds) with
    the bucket mask and the union correction, on sampled slots of two slices."""
    w = synth.WORKLOADS["64k"]
    _sampled_slices(w, [(0, 0), (7, 7)], slot_sample=2048, bucket_mask=True, union=True)


@pytest.mark.parametrize("scale,self_mask", [(None, False), (6.0, True), (40.0, True)])
def test_bucket_mask_tensor_core_attention_scales(scale, self_mask):
    """The tensor-core attention with the bucket mask (bf16, chunk 64): rows alone in their bucket
    see only themselves; at scale 40 the Cauchy-Schwarz shift underflows and the exact-maximum path
    (with the bucket mask) takes over."""
    w = synth.small_workload("bucket_tc_scale", 2, 2, 4096, 128, "bf16", 256, 64, 2)
    qk, v, R = synth.make_inputs(w, seed=33)
    qk_d, v_d, R_d = qk.to(DEV), v.to(DEV), R.to(DEV)
    b, _ = lsh.lsh_hash(qk_d, R_d, w.n_buckets)
    perm, _, _, _ = lsh.lsh_sort_permute(b, w.n_buckets)
    o, l = lsh.lsh_chunk_attend(qk_d, v_d, perm, w.chunk, self_mask=self_mask, buckets=b, bucket_mask=True,
                                scale=scale)
    torch.cuda.synchronize()
    assert lsh.lsh_get_device_status() == 0
    parity.check_attend(qk, v, perm, w.chunk, self_mask, scale, o, l, w.torch_dtype, g_buckets=b)


@pytest.mark.slow
def test_64k_workload_bucket_mask_sampled_slices():
    """The full-size launch with the bucket mask alone (tensor-core path), sampled slots of two slices."""
    w = synth.WORKLOADS["64k"]
    _sampled_slices(w, [(0, 0), (7, 7)], slot_sample=2048, bucket_mask=True)



@pytest.mark.parametrize("D,n_buckets,L", [(64, 4096, 1000), (128, 1536, 777), (64, 16384, 300),
                                           (128, 64, 1000), (64, 64, 777)])
def test_hash_streamed_and_narrow_projection(D, n_buckets, L):
    """The tensor-core hash's edge layouts of R[round]: bucket counts whose projection does not fit
    in shared memory (D * n_buckets > 128 K elements; R streams in 256-column chunks through a ring
    for every 128-row tile) and 64 buckets (32 columns, copied into a zero-padded 64-column tile,
    one epilogue part).  Buckets bit-exact against the float64 oracle except flagged rows, ragged
    row counts, several rounds.  The flag-free instantiation (the one the bench times; for rounds of
    4096 columns or more it takes the group-maximum fast path) is checked against the oracle the
    same way, with the flags of the flagged call, and agrees with the flagged call on every row
    that is not a near tie."""
    w = synth.small_workload("stream", 1, 2, L, D, "bf16", n_buckets, 64 if L % 64 == 0 else 1, 3)
    qk, v, R = synth.make_inputs(w, seed=21)
    qk_d, R_d = qk.to(DEV), R.to(DEV)
    b, nt = lsh.lsh_hash(qk_d, R_d, w.n_buckets)
    b_nf, _ = lsh.lsh_hash(qk_d, R_d, w.n_buckets, with_near_tie=False)
    assert lsh.lsh_get_device_status() == 0
    parity.check_hash(qk, R, w.n_buckets, b, nt, 1e-2)
    parity.check_hash(qk, R, w.n_buckets, b_nf, nt, 1e-2)
    clear = nt == 0
    assert torch.equal(b[clear], b_nf[clear])


def test_wide_round_hash_fast_path_at_the_1m_shape():
    """The flag-free hash at the 1M workload's projection (D 64, 16384 buckets: 8192 columns per
    round, the group-maximum fast path) on 32768 rows of one head: bit-exact against the float64
    oracle except near ties (flags from the flagged instantiation)."""
    w = synth.small_workload("wide", 1, 1, 32768, 64, "bf16", 16384, 64, 4)
    qk, v, R = synth.make_inputs(w, seed=5)
    qk_d, R_d = qk.to(DEV), R.to(DEV)
    b, nt = lsh.lsh_hash(qk_d, R_d, w.n_buckets)
    b_nf, _ = lsh.lsh_hash(qk_d, R_d, w.n_buckets, with_near_tie=False)
    assert lsh.lsh_get_device_status() == 0
    parity.check_hash(qk, R, w.n_buckets, b_nf, nt, 1e-2)
    clear = nt == 0
    assert torch.equal(b[clear], b_nf[clear])


@pytest.mark.parametrize("groups,kw", [(3, dict()), (1, dict()), (5, dict(bucket_mask=True, union=True)),
                                       (2, dict(causal=True))])
def test_host_pipeline_equals_device_call(groups, kw):
    """lsh_attention_host (host buffers, runs of slices on three streams) gives exactly the
    device-resident lsh_attention result: each (b, h) slice is an independent problem."""
    w = synth.small_workload("host_pipe", 2, 3, 2048, 128, "bf16", 64, 64, 3)
    qk, v, R = synth.make_inputs(w, seed=4)
    ref = lsh.lsh_attention(qk.cuda(), v.cuda(), R.cuda(), w.n_buckets, w.chunk, **kw)
    qk_h, v_h, R_h = qk.pin_memory(), v.pin_memory(), R.pin_memory()
    out_h = torch.empty_like(qk_h).pin_memory()
    state = {}
    for _ in range(2):  # the second call reuses the buffers and streams
        out_h.zero_()
        lsh.lsh_attention_host(qk_h, v_h, R_h, w.n_buckets, w.chunk, out_h, groups=groups, state=state, **kw)
        torch.cuda.synchronize()
        assert lsh.lsh_get_device_status() == 0
        assert torch.equal(out_h, ref.cpu())
