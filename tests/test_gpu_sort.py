"""The tiled counting sort (segments longer than 65536 positions or with more than 1024 buckets)
against an independent stable sort of the bucket ids.

The path counts per tile, scans each segment's counters in chunks, and scatters each tile with one
warp.  The shapes reach every regime:
- the scatter's running offsets in shared memory (at most 2048 buckets) or in the scanned counters
  in global memory;
- the count in shared memory (at most 16384 buckets) or in global memory;
- one or several scan chunks per segment, and a ragged last tile.
The reference is torch's stable argsort, a library sort, which is the plain definition of the step:
perm lists the positions of each segment ordered by (bucket, position).
"""

import pytest
import torch

import lsh_attention_hash_b200 as lsh

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("shape,n_buckets", [
    ((1, 1, 2, 70000), 64),        # shared-memory count and scatter, ragged last tile
    ((2, 2, 1, 50000), 2048),      # more than 1024 buckets, shared-memory scatter at its limit
    ((1, 2, 1, 100000), 4096),     # scatter on the global counters, several scan chunks per segment
    ((1, 1, 3, 300000), 16384),    # the 1M workload's bucket count, shared-memory count
    ((1, 1, 1, 300000), 32768),    # global-memory count and scatter
])
@pytest.mark.parametrize("skew", [False, True])
def test_tiled_sort_equals_stable_argsort(shape, n_buckets, skew):
    g = torch.Generator(device="cpu").manual_seed(n_buckets + (7 if skew else 0))
    hi = max(2, n_buckets // 64) if skew else n_buckets  # skewed: every id in a few buckets
    buckets = torch.randint(0, hi, shape, generator=g, dtype=torch.int32).to(DEV)
    assert lsh.lsh_get_device_status() == 0
    perm, inv, _, _ = lsh.lsh_sort_permute(buckets, n_buckets, want_inv=True)
    torch.cuda.synchronize()
    assert lsh.lsh_get_device_status() == 0
    ref = torch.argsort(buckets, dim=-1, stable=True).to(torch.int32)
    assert torch.equal(perm, ref)
    idx = torch.arange(shape[-1], device=DEV, dtype=torch.int64).expand(shape)
    assert torch.equal(torch.gather(inv.long(), -1, perm.long()), idx)
