"""Thin ctypes binding of liblsh_attention_hash.so (argument marshalling only).

Each function here has the name of the C entry point it calls, checks that the
tensors it forwards are contiguous CUDA tensors of the right dtype and shape
(so that no host pointer ever reaches a kernel), allocates missing outputs
with torch, and raises ``LSHError`` on a non-zero status.  All arithmetic
happens in the library's CUDA kernels; there is no CPU fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB = None

LSH_F32, LSH_BF16 = 0, 1
_DT = {torch.float32: LSH_F32, torch.bfloat16: LSH_BF16}
_STATUS = ["LSH_OK", "LSH_ERR_INVALID_ARG", "LSH_ERR_SHAPE", "LSH_ERR_DTYPE", "LSH_ERR_ALIGN",
           "LSH_ERR_WORKSPACE", "LSH_ERR_CUDA", "LSH_ERR_TIMEOUT", "LSH_ERR_UNSUPPORTED"]


class LSHError(RuntimeError):
    def __init__(self, code: int, where: str):
        name = _STATUS[code] if 0 <= code < len(_STATUS) else f"status {code}"
        super().__init__(f"{where}: {name}")
        self.code = code


def library_path() -> str:
    return os.path.join(_PKG, "liblsh_attention_hash.so")


_c_int, _c_size, _c_float, _vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p
_SIGS = {
    "lsh_abi_version": (_c_int, []),
    "lsh_status_string": (ctypes.c_char_p, [_c_int]),
    "lsh_hash": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _c_int, _c_int, _vp, _vp, _vp]),
    "lsh_sort_workspace_bytes": (_c_size, [_c_int] * 5),
    "lsh_sort_permute": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp,
                                  _c_int, _c_int, _vp, _vp, _vp, _c_size, _vp]),
    "lsh_sort_permute_noalloc": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "lsh_chunk_attend": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp,
                                  _vp, _vp, _c_int, _c_int, _c_float, _vp, _c_int, _vp, _vp]),
    "lsh_combine_rounds": (_c_int, [_vp, _c_int, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp,
                                    _c_int, _vp, _vp]),
    "lsh_chunk_attend_backward": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp,
                                           _c_int, _c_int, _c_float, _vp, _vp, _vp, _c_int, _vp, _vp, _vp]),
    "lsh_get_device_status": (_c_int, [_vp]),
}


def load_library():
    """Loads the CUDA library (once).  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m lsh_attention_hash_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _dt(t):
    if t.dtype not in _DT:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return _DT[t.dtype]


def _check(code, where):
    if code != 0:
        raise LSHError(code, where)


def lsh_hash(qk, R, n_buckets, *, buckets=None, near_tie=None, with_near_tie=True, stream=None):
    """Buckets [B,H,n_rounds,L] int32 (and near-tie flags uint8) of every row, all rounds."""
    lib = load_library()
    _need(qk, "qk")
    B, H, L, D = qk.shape
    _need(R, "R", qk.dtype)
    n_rounds = R.shape[0]
    if tuple(R.shape) != (n_rounds, D, n_buckets // 2):
        raise ValueError("R must be [n_rounds, D, n_buckets // 2]")
    shape = (B, H, n_rounds, L)
    if buckets is None:
        buckets = torch.empty(shape, dtype=torch.int32, device=qk.device)
    _need(buckets, "buckets", torch.int32, shape)
    if near_tie is None and with_near_tie:
        near_tie = torch.empty(shape, dtype=torch.uint8, device=qk.device)
    if near_tie is not None:
        _need(near_tie, "near_tie", torch.uint8, shape)
    _check(lib.lsh_hash(_ptr(qk), _dt(qk), B, H, L, D, _ptr(R), n_rounds, n_buckets, _ptr(buckets),
                        _ptr(near_tie), _stream(stream)), "lsh_hash")
    return buckets, near_tie


def lsh_sort_workspace_bytes(B, H, L, n_rounds, n_buckets):
    return int(load_library().lsh_sort_workspace_bytes(B, H, L, n_rounds, n_buckets))


def lsh_sort_permute(buckets, n_buckets, *, perm=None, inv=None, want_inv=False, qk=None, v=None,
                     qk_sorted=None, v_sorted=None, workspace=None, stream=None):
    """perm (and optionally inv and the gathered sorted rows) of every (b, h, round) segment.

    Returns (perm, inv, qk_sorted, v_sorted); absent outputs are None.
    """
    lib = load_library()
    _need(buckets, "buckets", torch.int32)
    B, H, n_rounds, L = buckets.shape
    shape = tuple(buckets.shape)
    dev = buckets.device
    if perm is None:
        perm = torch.empty(shape, dtype=torch.int32, device=dev)
    _need(perm, "perm", torch.int32, shape)
    if inv is None and want_inv:
        inv = torch.empty(shape, dtype=torch.int32, device=dev)
    if inv is not None:
        _need(inv, "inv", torch.int32, shape)
    dtype_code, D = LSH_BF16, 8
    if qk is not None or v is not None:
        _need(qk, "qk")
        _need(v, "v", qk.dtype, qk.shape)
        D = qk.shape[-1]
        dtype_code = _dt(qk)
        sshape = (B, H, n_rounds, L, D)
        if qk_sorted is None:
            qk_sorted = torch.empty(sshape, dtype=qk.dtype, device=dev)
        if v_sorted is None:
            v_sorted = torch.empty(sshape, dtype=qk.dtype, device=dev)
        _need(qk_sorted, "qk_sorted", qk.dtype, sshape)
        _need(v_sorted, "v_sorted", qk.dtype, sshape)
    need = lsh_sort_workspace_bytes(B, H, L, n_rounds, n_buckets)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8)
    _check(lib.lsh_sort_permute(_ptr(buckets), B, H, L, n_rounds, n_buckets, _ptr(perm), _ptr(inv),
                                _ptr(qk), _ptr(v), dtype_code, D, _ptr(qk_sorted), _ptr(v_sorted),
                                _ptr(workspace), workspace.numel(), _stream(stream)), "lsh_sort_permute")
    return perm, inv, qk_sorted, v_sorted


def lsh_sort_permute_noalloc(buckets, n_buckets, *, perm=None, inv=None, want_inv=False, stream=None):
    """perm (and optionally inv) using the library's own static scratch instead of a workspace.

    For callers that cannot provide device scratch memory; raises LSHError
    (LSH_ERR_WORKSPACE) when the sizes need more than the library's 16 MiB.
    Returns (perm, inv).
    """
    lib = load_library()
    _need(buckets, "buckets", torch.int32)
    B, H, n_rounds, L = buckets.shape
    shape = tuple(buckets.shape)
    if perm is None:
        perm = torch.empty(shape, dtype=torch.int32, device=buckets.device)
    _need(perm, "perm", torch.int32, shape)
    if inv is None and want_inv:
        inv = torch.empty(shape, dtype=torch.int32, device=buckets.device)
    if inv is not None:
        _need(inv, "inv", torch.int32, shape)
    _check(lib.lsh_sort_permute_noalloc(_ptr(buckets), B, H, L, n_rounds, n_buckets, _ptr(perm), _ptr(inv),
                                        _stream(stream)), "lsh_sort_permute_noalloc")
    return perm, inv


def lsh_chunk_attend(qk, v, perm, chunk, *, self_mask=True, causal=False, buckets=None, bucket_mask=False,
                     union=False, scale=None, qk_sorted=None, v_sorted=None, out_dtype=None, out_rounds=None,
                     lse=None, stream=None):
    """Per-round outputs [B,H,n_rounds,L,D] and log-sum-exp [B,H,n_rounds,L] in original order.

    ``causal``: keys after the query's original position are not admissible.
    ``bucket_mask`` (needs ``buckets`` from ``lsh_hash``): keys outside the query's bucket
    are not admissible.  ``union`` (with ``bucket_mask``): each logit is lowered by the log
    of the number of rounds in which query and key share a bucket.
    """
    lib = load_library()
    _need(qk, "qk")
    _need(v, "v", qk.dtype, qk.shape)
    B, H, L, D = qk.shape
    _need(perm, "perm", torch.int32)
    n_rounds = perm.shape[2]
    _need(perm, "perm", torch.int32, (B, H, n_rounds, L))
    if union and not bucket_mask:
        raise ValueError("union needs bucket_mask")
    if bucket_mask:
        if buckets is None:
            raise ValueError("bucket_mask needs buckets")
        _need(buckets, "buckets", torch.int32, (B, H, n_rounds, L))
    if qk_sorted is not None or v_sorted is not None:
        _need(qk_sorted, "qk_sorted", qk.dtype, (B, H, n_rounds, L, D))
        _need(v_sorted, "v_sorted", qk.dtype, (B, H, n_rounds, L, D))
    out_dtype = qk.dtype if out_dtype is None else out_dtype
    if out_rounds is None:
        out_rounds = torch.empty((B, H, n_rounds, L, D), dtype=out_dtype, device=qk.device)
    _need(out_rounds, "out_rounds", out_dtype, (B, H, n_rounds, L, D))
    if lse is None:
        lse = torch.empty((B, H, n_rounds, L), dtype=torch.float32, device=qk.device)
    _need(lse, "lse", torch.float32, (B, H, n_rounds, L))
    sc = 0.0 if scale is None else float(scale)
    mask = (1 if self_mask else 0) | (2 if causal else 0) | (4 if bucket_mask else 0) | (8 if union else 0)
    _check(lib.lsh_chunk_attend(_ptr(qk), _ptr(v), _dt(qk), B, H, L, D, n_rounds, _ptr(perm),
                                _ptr(buckets) if bucket_mask else None, _ptr(qk_sorted), _ptr(v_sorted),
                                int(chunk), mask, sc,
                                _ptr(out_rounds), _DT[out_dtype], _ptr(lse), _stream(stream)),
           "lsh_chunk_attend")
    return out_rounds, lse


def lsh_combine_rounds(out_rounds, lse, *, out_dtype=None, out=None, lse_out=None, want_lse=True,
                       stream=None):
    """Round merge: (out [B,H,L,D], LSE [B,H,L] or None)."""
    lib = load_library()
    _need(out_rounds, "out_rounds")
    B, H, n_rounds, L, D = out_rounds.shape
    _need(lse, "lse", torch.float32, (B, H, n_rounds, L))
    out_dtype = out_rounds.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((B, H, L, D), dtype=out_dtype, device=out_rounds.device)
    _need(out, "out", out_dtype, (B, H, L, D))
    if lse_out is None and want_lse:
        lse_out = torch.empty((B, H, L), dtype=torch.float32, device=out_rounds.device)
    if lse_out is not None:
        _need(lse_out, "lse_out", torch.float32, (B, H, L))
    _check(lib.lsh_combine_rounds(_ptr(out_rounds), _dt(out_rounds), _ptr(lse), B, H, L, D, n_rounds,
                                  _ptr(out), _DT[out_dtype], _ptr(lse_out), _stream(stream)),
           "lsh_combine_rounds")
    return out, lse_out


def lsh_chunk_attend_backward(qk, v, perm, chunk, out, lse, dout, *, self_mask=True, causal=False, buckets=None,
                              bucket_mask=False, union=False, scale=None, dqk=None, dv=None, stream=None):
    """Gradients (dqk, dv) [B,H,L,D] float32 of sum(dout * out) for the merged output.

    ``out`` and ``lse`` are the merged output and LSE of the forward (``lsh_combine_rounds``);
    ``perm``, ``buckets``, the masks and ``scale`` must be the forward's.
    """
    lib = load_library()
    _need(qk, "qk")
    _need(v, "v", qk.dtype, qk.shape)
    B, H, L, D = qk.shape
    _need(perm, "perm", torch.int32)
    n_rounds = perm.shape[2]
    _need(perm, "perm", torch.int32, (B, H, n_rounds, L))
    _need(out, "out", None, (B, H, L, D))
    _need(dout, "dout", out.dtype, (B, H, L, D))
    _need(lse, "lse", torch.float32, (B, H, L))
    if union and not bucket_mask:
        raise ValueError("union needs bucket_mask")
    if bucket_mask:
        if buckets is None:
            raise ValueError("bucket_mask needs buckets")
        _need(buckets, "buckets", torch.int32, (B, H, n_rounds, L))
    if dqk is None:
        dqk = torch.empty((B, H, L, D), dtype=torch.float32, device=qk.device)
    if dv is None:
        dv = torch.empty((B, H, L, D), dtype=torch.float32, device=qk.device)
    _need(dqk, "dqk", torch.float32, (B, H, L, D))
    _need(dv, "dv", torch.float32, (B, H, L, D))
    mask = (1 if self_mask else 0) | (2 if causal else 0) | (4 if bucket_mask else 0) | (8 if union else 0)
    sc = 0.0 if scale is None else float(scale)
    _check(lib.lsh_chunk_attend_backward(_ptr(qk), _ptr(v), _dt(qk), B, H, L, D, n_rounds, _ptr(perm),
                                         _ptr(buckets) if bucket_mask else None, int(chunk), mask, sc, _ptr(out),
                                         _ptr(lse), _ptr(dout), _dt(out), _ptr(dqk), _ptr(dv), _stream(stream)),
           "lsh_chunk_attend_backward")
    return dqk, dv


def lsh_get_device_status(stream=None) -> int:
    """Synchronises the stream; returns and clears the device status word (0 = LSH_OK)."""
    return int(load_library().lsh_get_device_status(_stream(stream)))


def lsh_attention(qk, v, R, n_buckets, chunk, *, self_mask=True, causal=False, bucket_mask=False, union=False,
                  scale=None, stream=None, return_all=False, bufs=None, check=False):
    """The whole forward pass: hash, sort, chunk attention, round merge (four C-ABI calls).

    ``bufs`` may hold preallocated outputs (keys: buckets, near_tie, perm, workspace,
    out_rounds, lse_rounds, out, lse) so that repeated calls allocate nothing.

    The calls are asynchronous.  Errors that the kernels detect while they run (an
    exhausted bounded wait, a bucket id out of range) are recorded in the device
    status word, not returned: with ``check=True`` the stream is synchronised and a
    non-zero status raises ``LSHError``; otherwise the caller reads it with
    ``lsh_get_device_status`` before trusting the outputs.
    """
    b = bufs or {}
    buckets, near = lsh_hash(qk, R, n_buckets, buckets=b.get("buckets"), near_tie=b.get("near_tie"),
                             with_near_tie=return_all or "near_tie" in b, stream=stream)
    perm, _, _, _ = lsh_sort_permute(buckets, n_buckets, perm=b.get("perm"), workspace=b.get("workspace"),
                                     stream=stream)
    o, lse = lsh_chunk_attend(qk, v, perm, chunk, self_mask=self_mask, causal=causal, buckets=buckets,
                              bucket_mask=bucket_mask, union=union, scale=scale,
                              out_rounds=b.get("out_rounds"), lse=b.get("lse_rounds"), stream=stream)
    out, lse_out = lsh_combine_rounds(o, lse, out=b.get("out"), lse_out=b.get("lse"),
                                      want_lse=return_all or "lse" in b, stream=stream)
    if check:
        _check(lsh_get_device_status(stream), "lsh_attention (device status)")
    if return_all:
        return {"buckets": buckets, "near_tie": near, "perm": perm, "o_rounds": o, "lse_rounds": lse,
                "out": out, "lse": lse_out}
    return out


def lsh_attention_host(qk_h, v_h, R, n_buckets, chunk, out_h, *, groups=8, self_mask=True, causal=False,
                       bucket_mask=False, union=False, scale=None, stream=None, state=None):
    """The forward pass on host data: ``qk_h``, ``v_h`` [B, H, L, D] in pinned host memory, the
    merged output written into ``out_h`` (pinned, same shape); ``R`` on the device or pinned host.

    The B*H (b, h) slices are independent problems, processed in ``groups`` contiguous runs.
    Three CUDA streams overlap the host-to-device copy of run g + 1, the four library calls on
    run g and the device-to-host copy of run g - 1 (two device buffers per run tensor, so PCIe
    carries both directions while the kernels run).  The work starts after what is already
    queued on ``stream`` (default: the current stream) and ``stream`` waits for all of it, so
    events recorded on ``stream`` around the call time the copies and the kernels together.
    ``state`` (a dict) keeps the device buffers and streams between calls; each run's results
    are those of ``lsh_attention`` on its slices.
    """
    for t, nm in ((qk_h, "qk_h"), (v_h, "v_h"), (out_h, "out_h")):
        if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_pinned() or not t.is_contiguous():
            raise ValueError(f"{nm} must be a contiguous pinned host tensor")
        if t.dtype != qk_h.dtype or t.shape != qk_h.shape:
            raise ValueError(f"{nm} must match qk_h ({qk_h.dtype}, {tuple(qk_h.shape)})")
    B, H, L, D = qk_h.shape
    dev = R.device if R.is_cuda else torch.device("cuda", torch.cuda.current_device())
    main = stream if stream is not None else torch.cuda.current_stream(dev)
    n = B * H
    G = max(1, min(int(groups), n))
    bounds = [(n * g) // G for g in range(G + 1)]
    m_max = max(bounds[g + 1] - bounds[g] for g in range(G))
    st = state if state is not None else {}
    key = (n, L, D, qk_h.dtype, tuple(R.shape), n_buckets, G, str(dev))
    if st.get("key") != key:
        st.clear()
        st["key"] = key
        st["qk"] = [torch.empty((1, m_max, L, D), dtype=qk_h.dtype, device=dev) for _ in range(2)]
        st["v"] = [torch.empty((1, m_max, L, D), dtype=qk_h.dtype, device=dev) for _ in range(2)]
        st["out"] = [torch.empty((1, m_max, L, D), dtype=qk_h.dtype, device=dev) for _ in range(2)]
        st["R"] = torch.empty(R.shape, dtype=R.dtype, device=dev)
        st["bufs"] = alloc_buffers(1, m_max, L, D, R.shape[0], n_buckets, qk_h.dtype, dev)
        st["streams"] = [torch.cuda.Stream(dev) for _ in range(3)]
    qf, vf, of = (t.view(1, n, L, D) for t in (qk_h, v_h, out_h))
    if G == 1:  # one run: nothing to overlap, everything in order on the caller's stream
        with torch.cuda.stream(main):
            dq, dv, do = st["qk"][0], st["v"][0], st["out"][0]
            dq.copy_(qf, non_blocking=True)
            dv.copy_(vf, non_blocking=True)
            Rd = R if R.is_cuda else st["R"].copy_(R, non_blocking=True)
            bufs = dict(st["bufs"], out=do)
            lsh_attention(dq, dv, Rd, n_buckets, chunk, self_mask=self_mask, causal=causal,
                          bucket_mask=bucket_mask, union=union, scale=scale, stream=main, bufs=bufs)
            of.copy_(do, non_blocking=True)
        return out_h
    s_in, s_run, s_out = st["streams"]
    start = torch.cuda.Event()
    start.record(main)
    for s_ in (s_in, s_run, s_out):
        s_.wait_event(start)
    if R.is_cuda:
        Rd = R
    else:
        with torch.cuda.stream(s_in):
            st["R"].copy_(R, non_blocking=True)
        Rd = st["R"]
    run_done, out_done = [None] * G, [None] * G
    for g in range(G):
        a, b = bounds[g], bounds[g + 1]
        k, m = g % 2, b - a
        dq, dv, do = st["qk"][k][:, :m], st["v"][k][:, :m], st["out"][k][:, :m]
        if g >= 2:  # buffer pair k was last read by run g - 2's calls
            s_in.wait_event(run_done[g - 2])
        with torch.cuda.stream(s_in):
            dq.copy_(qf[:, a:b], non_blocking=True)
            dv.copy_(vf[:, a:b], non_blocking=True)
        in_done = torch.cuda.Event()
        in_done.record(s_in)
        s_run.wait_event(in_done)
        if g >= 2:  # output buffer k was last read by run g - 2's device-to-host copy
            s_run.wait_event(out_done[g - 2])
        bufs = {nm: (t if nm == "workspace" else t[:, :m]) for nm, t in st["bufs"].items()}
        bufs["out"] = do
        lsh_attention(dq, dv, Rd, n_buckets, chunk, self_mask=self_mask, causal=causal, bucket_mask=bucket_mask,
                      union=union, scale=scale, stream=s_run, bufs=bufs)
        run_done[g] = torch.cuda.Event()
        run_done[g].record(s_run)
        s_out.wait_event(run_done[g])
        with torch.cuda.stream(s_out):
            of[:, a:b].copy_(do, non_blocking=True)
        out_done[g] = torch.cuda.Event()
        out_done[g].record(s_out)
    main.wait_event(out_done[G - 1])
    return out_h


def alloc_buffers(B, H, L, D, n_rounds, n_buckets, dtype, device, with_near_tie=False):
    """Preallocated buffers for ``lsh_attention`` (device memory through torch)."""
    ws = lsh_sort_workspace_bytes(B, H, L, n_rounds, n_buckets)
    bufs = {
        "buckets": torch.empty((B, H, n_rounds, L), dtype=torch.int32, device=device),
        "perm": torch.empty((B, H, n_rounds, L), dtype=torch.int32, device=device),
        "workspace": torch.empty(max(ws, 16), dtype=torch.uint8, device=device),
        "out_rounds": torch.empty((B, H, n_rounds, L, D), dtype=dtype, device=device),
        "lse_rounds": torch.empty((B, H, n_rounds, L), dtype=torch.float32, device=device),
        "out": torch.empty((B, H, L, D), dtype=dtype, device=device),
    }
    if with_near_tie:
        bufs["near_tie"] = torch.empty((B, H, n_rounds, L), dtype=torch.uint8, device=device)
    return bufs

