"""The allocation-free sort entry point, lsh_sort_permute_noalloc.

It serves callers that cannot give the library scratch memory (a plugin that
only receives its input and output buffers, a process whose device memory is
already reserved by another allocator, code that must not pay cudaMalloc's
synchronisation).  Instead of a caller workspace it uses a 16 MiB static
device array inside the library, which keeps the previous call's contents.

The test calls it through the C ABI twice in a row, on different inputs, for
every path of the sort (one CTA per segment with no scratch at all, as at the
64K workload; shared-memory histograms; global-memory counters that the call
must clear itself), and checks that every result is identical to the
workspace-based lsh_sort_permute.  Sizes beyond the static
array are rejected with LSH_ERR_WORKSPACE before any launch.  This file runs
last (pytest collects it after the others) and also passes on its own.
"""

import ctypes

import pytest
import torch

import lsh_attention_hash_b200 as lsh

pytestmark = pytest.mark.gpu
DEV = "cuda"
LSH_ERR_WORKSPACE = 5


def _buckets(shape, n_buckets, seed, skew=False):
    g = torch.Generator(device="cpu").manual_seed(seed)
    if skew:  # most ids in a few buckets
        b = torch.randint(0, max(2, n_buckets // 64), shape, generator=g, dtype=torch.int32)
    else:
        b = torch.randint(0, n_buckets, shape, generator=g, dtype=torch.int32)
    return b.to(DEV)


def _noalloc(buckets, n_buckets, perm, inv):
    lib = lsh.load_library()
    B, H, nr, L = buckets.shape
    return lib.lsh_sort_permute_noalloc(ctypes.c_void_p(buckets.data_ptr()), B, H, L, nr, n_buckets,
                                        ctypes.c_void_p(perm.data_ptr()), ctypes.c_void_p(inv.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("shape,n_buckets", [
    ((1, 2, 4, 65536), 1024),     # the 64K workload's segments: one CTA per segment, no scratch
    ((1, 1, 70000, 16), 16),      # more than 65535 segments (one CTA per segment)
    ((2, 3, 2, 70000), 64),       # counters in shared memory, ragged last tile
    ((1, 2, 1, 70000), 32768),    # counters in global memory: cleared by the call
])
def test_noalloc_sort_matches_workspace_sort_on_consecutive_calls(shape, n_buckets):
    for call, (seed, skew) in enumerate([(11, False), (12, True)]):
        b = _buckets(shape, n_buckets, seed, skew)
        ref_perm, ref_inv, _, _ = lsh.lsh_sort_permute(b, n_buckets, want_inv=True)
        perm = torch.full_like(b, -1)
        inv = torch.full_like(b, -1)
        assert _noalloc(b, n_buckets, perm, inv) == 0, f"call {call}"
        torch.cuda.synchronize()
        assert lsh.lsh_get_device_status() == 0
        assert torch.equal(perm, ref_perm), f"perm differs on call {call}"
        assert torch.equal(inv, ref_inv), f"inv differs on call {call}"


def test_noalloc_sort_rejects_sizes_beyond_its_scratch():
    # 64 segments x 16384 buckets x 16 tiles of 16384 positions = 16M counters > 4M
    lib = lsh.load_library()
    dummy = torch.zeros(16, dtype=torch.int32, device=DEV)
    p = ctypes.c_void_p(dummy.data_ptr())
    assert lib.lsh_sort_permute_noalloc(p, 8, 8, 262144, 1, 16384, p, None, None) == LSH_ERR_WORKSPACE
