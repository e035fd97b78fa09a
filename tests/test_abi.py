"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments before any launch."""

import ctypes
import os
import re

import pytest
import torch

import lsh_attention_hash_b200 as lsh
from lsh_attention_hash_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]

# codes from include/lsh_attention_hash.h
OK, INVALID, SHAPE, DTYPE, ALIGN, WORKSPACE, UNSUPPORTED = 0, 1, 2, 3, 4, 5, 8
F32, BF16 = 0, 1
A = 0x10000  # a 16-byte aligned non-null address that is never dereferenced (rejected before launch)


def declared_symbols():
    names = []
    for h in HEADERS:
        src = open(h).read()
        names += re.findall(r"LSH_API\s+[\w\s\*]+?\b(lsh_\w+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    return lsh.load_library()


def test_library_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert lib.lsh_abi_version() == 2


def _declared_param_counts():
    """Number of parameters of every LSH_API declaration (void counts as none)."""
    out = {}
    for h in HEADERS:
        src = open(h).read()
        for name, params in re.findall(r"LSH_API\s+[\w\s\*]+?\b(lsh_\w+)\s*\(([^)]*)\)", src):
            params = params.strip()
            out[name] = 0 if params in ("", "void") else len(params.split(","))
    return out


def test_binding_signatures_match_the_header():
    """The ctypes argument lists have as many entries as the C declarations have parameters, and
    every declared entry point has a binding signature."""
    from lsh_attention_hash_b200 import binding

    counts = _declared_param_counts()
    assert set(counts) == set(declared_symbols())
    for name, n in counts.items():
        assert name in binding._SIGS, name
        assert len(binding._SIGS[name][1]) == n, (name, len(binding._SIGS[name][1]), n)


def test_library_exports_nothing_undeclared(lib):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", lsh.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.split() and line.split()[-1].startswith("lsh_")}
    assert exported == set(declared_symbols()), exported ^ set(declared_symbols())


def test_status_strings(lib):
    assert lib.lsh_status_string(0) == b"LSH_OK"
    assert lib.lsh_status_string(7) == b"LSH_ERR_TIMEOUT"
    assert lib.lsh_status_string(99) == b"LSH_ERR_UNKNOWN"


def test_hash_rejects_bad_arguments_before_launch(lib):
    h = lib.lsh_hash
    assert h(A, 7, 1, 1, 64, 64, A, 1, 16, A, None, None) == DTYPE
    assert h(A, BF16, 1, 1, 64, 64, A, 1, 15, A, None, None) == SHAPE     # odd n_buckets
    assert h(A, BF16, 1, 1, 64, 64, A, 1, 0, A, None, None) == SHAPE
    assert h(A, BF16, 1, 1, 64, 60, A, 1, 16, A, None, None) == SHAPE     # D % 8
    assert h(A, BF16, 1, 1, 64, 512, A, 1, 16, A, None, None) == SHAPE    # D > 256
    assert h(A, BF16, 1, 1, 64, 64, A, 0, 16, A, None, None) == SHAPE     # no rounds
    assert h(None, BF16, 1, 1, 64, 64, A, 1, 16, A, None, None) == INVALID
    assert h(A, BF16, 1, 1, 64, 64, A, 1, 16, None, None, None) == INVALID
    assert h(A + 4, BF16, 1, 1, 64, 64, A, 1, 16, A, None, None) == ALIGN
    assert h(A, BF16, 1, 1, 64, 64, A, 1, 16, A, A + 1, None) == ALIGN
    assert h(A, BF16, 4096, 4096, 4096, 64, A, 64, 16, A, None, None) == SHAPE  # int32 index space
    assert h(A, BF16, 0, 1, 64, 64, A, 1, 16, A, None, None) == OK        # empty: no launch


def test_sort_rejects_bad_arguments_before_launch(lib):
    s = lib.lsh_sort_permute
    # one CTA per segment (L <= 65536, <= 1024 buckets) needs no workspace
    assert lib.lsh_sort_workspace_bytes(1, 1, 1024, 1, 16) == 0
    # more buckets: the count / scan / scatter sort and its workspace
    nb = 2048
    ws = lib.lsh_sort_workspace_bytes(1, 1, 1024, 1, nb)
    assert ws > 0
    assert s(A, 1, 1, 1024, 1, 15, A, None, None, None, BF16, 64, None, None, A, ws, None) == SHAPE
    assert s(None, 1, 1, 1024, 1, nb, A, None, None, None, BF16, 64, None, None, A, ws, None) == INVALID
    assert s(A, 1, 1, 1024, 1, nb, A, None, None, None, BF16, 64, None, None, None, 0, None) == WORKSPACE
    assert s(A, 1, 1, 1024, 1, nb, A, None, None, None, BF16, 64, None, None, A, ws - 4, None) == WORKSPACE
    assert s(A, 1, 1, 1024, 1, nb, A, None, None, None, BF16, 64, None, None, A + 8, ws, None) == ALIGN
    assert s(A, 1, 1, 1024, 1, nb, A, None, A, None, BF16, 64, None, None, A, ws, None) == INVALID  # half a gather
    assert s(A, 1, 1, 1024, 1, nb, A, A + 8, None, None, BF16, 64, None, None, A, ws, None) == ALIGN
    assert s(A, 0, 1, 1024, 1, nb, A, None, None, None, BF16, 64, None, None, None, 0, None) == OK


def test_attend_rejects_bad_arguments_before_launch(lib):
    f = lib.lsh_chunk_attend
    args = [A, A, BF16, 1, 1, 1024, 64, 1, A, None, None, None, 64, 1, 0.0, A, BF16, A, None]

    def call(**kw):
        a = list(args)
        names = ["qk", "v", "dtype", "B", "H", "L", "D", "nr", "perm", "bk", "qs", "vs", "chunk", "mask",
                 "scale", "out", "out_dtype", "lse", "stream"]
        for k, val in kw.items():
            a[names.index(k)] = val
        return f(*a)

    assert call(chunk=48) == SHAPE        # 1024 % 48 != 0
    assert call(chunk=0) == SHAPE
    assert call(chunk=2048) == SHAPE      # chunk > L
    assert call(mask=16) == INVALID       # bits beyond the four of lsh_mask
    assert call(mask=-1) == INVALID
    assert call(mask=1 | 4) == INVALID    # bucket mask without buckets
    assert call(mask=1 | 8, bk=A) == INVALID  # union without the bucket mask
    assert call(mask=1 | 4, bk=A + 4) == ALIGN
    assert call(mask=1 | 4 | 8, bk=A, L=0) == OK
    # the union's per-round bucket tables no longer fit in shared memory
    assert call(mask=1 | 4 | 8, bk=A, dtype=F32, out_dtype=F32, D=256, nr=600, chunk=32) == UNSUPPORTED
    assert call(out_dtype=5) == DTYPE
    assert call(qs=A) == INVALID          # sorted qk without sorted v
    assert call(lse=None) == INVALID
    assert call(out=A + 2) == ALIGN
    assert call(L=0) == OK


def test_backward_rejects_bad_arguments_before_launch(lib):
    f = lib.lsh_chunk_attend_backward
    args = [A, A, BF16, 1, 1, 1024, 64, 2, A, None, 64, 1, 0.0, A, A, A, BF16, A, A, None]
    names = ["qk", "v", "dtype", "B", "H", "L", "D", "nr", "perm", "bk", "chunk", "mask", "scale", "out",
             "lse", "dout", "out_dtype", "dqk", "dv", "stream"]

    def call(**kw):
        a = list(args)
        for k, val in kw.items():
            a[names.index(k)] = val
        return f(*a)

    assert call(dtype=3) == DTYPE
    assert call(out_dtype=3) == DTYPE
    assert call(chunk=48) == SHAPE
    assert call(D=60) == SHAPE
    assert call(nr=0) == SHAPE
    assert call(mask=16) == INVALID
    assert call(mask=1 | 4) == INVALID        # bucket mask without buckets
    assert call(mask=1 | 8, bk=A) == INVALID  # union without the bucket mask
    assert call(dout=None) == INVALID
    assert call(dqk=None) == INVALID
    assert call(lse=A + 4) == ALIGN
    assert call(dv=A + 8) == ALIGN
    assert call(mask=1 | 4 | 8, bk=A, D=256, nr=400) == UNSUPPORTED  # union tables beyond shared memory
    assert call(B=0) == OK                    # empty: no launch
    assert call(L=0) == OK


def test_combine_rejects_bad_arguments_before_launch(lib):
    c = lib.lsh_combine_rounds
    assert c(A, 9, A, 1, 1, 64, 64, 2, A, BF16, None, None) == DTYPE
    assert c(A, BF16, A, 1, 1, 64, 64, 0, A, BF16, None, None) == SHAPE
    assert c(None, BF16, A, 1, 1, 64, 64, 2, A, BF16, None, None) == INVALID
    assert c(A, BF16, A, 1, 1, 64, 64, 2, A, BF16, A + 4, None) == ALIGN


def test_binding_refuses_host_tensors():
    qk = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    R = torch.zeros(1, 64, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        lsh.lsh_hash(qk, R, 16)


def test_sort_workspace_formula_bounds(lib):
    # whole segments in one CTA need none
    for (B, H, L, nr, nb) in [(8, 8, 65536, 8, 1024), (1, 1, 1024, 1, 16), (8, 8, 16384, 4, 256)]:
        assert lib.lsh_sort_workspace_bytes(B, H, L, nr, nb) == 0
    # radix sort: digit-major counters per 4096-element tile, the scan chunks' sums and the valid
    # counts, and with two passes (more than 256 buckets) the first pass's ids and positions
    for (B, H, L, nr, nb) in [(1, 8, 1 << 20, 4, 16384), (1, 1, 1024, 1, 2048), (2, 2, 70000, 2, 64)]:
        ws = lib.lsh_sort_workspace_bytes(B, H, L, nr, nb)
        segs = B * H * nr
        counters = segs * 256 * ((L + 4095) // 4096)
        pairs = 2 * segs * L if nb > 256 else 0
        assert 4 * (counters + pairs) < ws <= 4 * (counters + pairs + 66 * segs + 3)
