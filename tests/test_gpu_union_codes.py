"""The union correction's bucket codes on the tensor-core path (bf16, D 128, chunk 64).

The tensor-core kernels compare each round's buckets as fp16 codes (0x0400 + bucket).  An
order-preserving relabelling of the buckets leaves the sorted order, every bucket test and every
shared-round count unchanged, so the forward and backward outputs must stay bit-identical when the
ids are moved to the top of the codable range.  A bucket id without a code (30720 and up) is an
error that the device status word reports, without a fault.
"""

import pytest
import torch

import lsh_attention_hash_b200 as lsh

pytestmark = pytest.mark.gpu
DEV = "cuda"
MAX_CODABLE = 30719
UNSUPPORTED = 8  # LSH_ERR_UNSUPPORTED


def _inputs(seed, B=1, H=2, L=512, D=128, n_rounds=3, n_buckets=16):
    g = torch.Generator().manual_seed(seed)
    qk = torch.randn(B, H, L, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, L, D, generator=g).to(torch.bfloat16)
    dout = torch.randn(B, H, L, D, generator=g).to(torch.bfloat16)
    buckets = torch.randint(0, n_buckets, (B, H, n_rounds, L), generator=g, dtype=torch.int32)
    return qk, v, dout, buckets


def _run(qk, v, dout, buckets, causal=False):
    perm = torch.argsort(buckets, dim=-1, stable=True).to(torch.int32).to(DEV)
    qk_d, v_d, bk = qk.to(DEV), v.to(DEV), buckets.to(DEV)
    o_r, lse_r = lsh.lsh_chunk_attend(qk_d, v_d, perm, 64, buckets=bk, bucket_mask=True, union=True, causal=causal)
    out, lse = lsh.lsh_combine_rounds(o_r, lse_r)
    dqk, dv = lsh.lsh_chunk_attend_backward(qk_d, v_d, perm, 64, out, lse, dout.to(DEV), buckets=bk,
                                            bucket_mask=True, union=True, causal=causal)
    torch.cuda.synchronize()
    return [t.cpu() for t in (o_r, lse_r, dqk, dv)]


@pytest.mark.parametrize("causal", [False, True])
def test_relabelled_buckets_give_identical_results(causal):
    qk, v, dout, buckets = _inputs(7)
    assert lsh.lsh_get_device_status() == 0
    base = _run(qk, v, dout, buckets, causal)
    assert lsh.lsh_get_device_status() == 0
    # same order and equality structure, ids at the top of the codable range
    shifted = buckets + (MAX_CODABLE - int(buckets.max()))
    assert int(shifted.max()) == MAX_CODABLE
    moved = _run(qk, v, dout, shifted, causal)
    assert lsh.lsh_get_device_status() == 0
    for a, b in zip(base, moved):
        assert torch.equal(a, b)
    # the union correction is active: without it the outputs differ
    perm = torch.argsort(buckets, dim=-1, stable=True).to(torch.int32).to(DEV)
    o_plain, _ = lsh.lsh_chunk_attend(qk.to(DEV), v.to(DEV), perm, 64, buckets=buckets.to(DEV), bucket_mask=True,
                                      causal=causal)
    torch.cuda.synchronize()
    assert not torch.equal(o_plain.cpu(), base[0])


def test_bucket_without_code_reports_unsupported():
    qk, v, dout, buckets = _inputs(8)
    assert lsh.lsh_get_device_status() == 0
    bad = buckets.clone()
    bad[0, 1, 2, 100] = MAX_CODABLE + 1
    perm = torch.argsort(bad, dim=-1, stable=True).to(torch.int32).to(DEV)
    lsh.lsh_chunk_attend(qk.to(DEV), v.to(DEV), perm, 64, buckets=bad.to(DEV), bucket_mask=True, union=True)
    torch.cuda.synchronize()
    assert lsh.lsh_get_device_status() == UNSUPPORTED
    assert lsh.lsh_get_device_status() == 0  # read and cleared
