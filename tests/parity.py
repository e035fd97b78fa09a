"""Stage-wise comparison of the CUDA path with the float64 oracle.

Rules (the same for every workload):
  * buckets: bit-exact, except rows flagged as near ties (top-two gap < 1e-5
    relative) by either side; the excluded set is the union of both flags;
  * perm: bit-exact against the oracle's sort of the GPU's own buckets (a
    flagged row that hashed differently moves its neighbours, so each stage is
    checked on the previous stage's GPU output);
  * per-round outputs, log-sum-exp and the merged output: max-abs error within
    TOL[dtype] against the oracle run on the GPU's perm / per-round outputs.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import oracle_attend, oracle_attend_slots, oracle_combine, oracle_hash, oracle_sort

# max-abs tolerances on attention outputs (fp32 accumulation everywhere)
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def np_(t):
    return t.detach().cpu().numpy() if isinstance(t, torch.Tensor) else np.asarray(t)


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check_hash(qk, R, n_buckets, g_buckets, g_near, max_flag_frac=1e-3):
    """Returns (#mismatch, #flagged) after asserting mismatches are all flagged."""
    o_b, o_f = oracle_hash(qk, R, n_buckets)
    g_b = np_(g_buckets)
    g_f = np_(g_near).astype(bool)
    excl = o_f | g_f
    mism = g_b != o_b
    assert not (mism & ~excl).any(), f"{int((mism & ~excl).sum())} unflagged bucket mismatches"
    assert excl.mean() <= max_flag_frac, f"flagged fraction {excl.mean():.2e}"
    return int(mism.sum()), int(excl.sum())


def check_sort(g_buckets, g_perm):
    o_p = oracle_sort(np_(g_buckets))
    assert np.array_equal(o_p, np_(g_perm)), "perm differs from the oracle's sort of the same buckets"


def check_attend(qk, v, g_perm, chunk, self_mask, scale, g_o, g_lse, dtype, causal=False, g_buckets=None,
                 union=False):
    """g_buckets (the GPU's buckets), when given, selects the bucket-equality mask."""
    o, lse = oracle_attend(f64(qk), f64(v), np_(g_perm), chunk, self_mask, scale, causal,
                           None if g_buckets is None else np_(g_buckets), union)
    err_o = float(np.max(np.abs(o - f64(g_o)))) if o.size else 0.0
    err_l = float(np.max(np.abs(lse - f64(g_lse)))) if lse.size else 0.0
    tol = TOL[dtype]
    assert err_o <= tol, f"per-round output max-abs error {err_o:.3e} > {tol}"
    assert err_l <= tol, f"per-round lse max-abs error {err_l:.3e} > {tol}"
    return err_o, err_l


def check_combine(g_o, g_lse, g_out, g_lse_out, dtype):
    out, big = oracle_combine(f64(g_o), f64(g_lse))
    err = float(np.max(np.abs(out - f64(g_out)))) if out.size else 0.0
    tol = TOL[dtype]
    assert err <= tol, f"merged output max-abs error {err:.3e} > {tol}"
    if g_lse_out is not None and big.size:
        err_l = float(np.max(np.abs(big - f64(g_lse_out))))
        assert err_l <= tol, f"merged lse max-abs error {err_l:.3e} > {tol}"
    return err


def check_slice_rounds(qk_bh, v_bh, g_perm_bh, chunk, self_mask, scale, g_o_bh, g_lse_bh, dtype,
                       slots=None, g_buckets_bh=None, union=False):
    """Per-round attention of one (b, h) slice at full size (all rounds, optional slot sample).

    g_buckets_bh ([n_rounds, L], the GPU's), when given, selects the bucket-equality mask."""
    n_rounds, L = g_perm_bh.shape
    bk = None if g_buckets_bh is None else np_(g_buckets_bh)
    worst = 0.0
    for r in range(n_rounds):
        ss = np.arange(L) if slots is None else np.asarray(slots)
        pos, o, lse = oracle_attend_slots(f64(qk_bh), f64(v_bh), np_(g_perm_bh[r]), chunk, ss, self_mask, scale,
                                          bucket_seg=None if bk is None else bk[r],
                                          union_buckets=bk if union else None)
        go = f64(g_o_bh[r])[pos]
        gl = f64(g_lse_bh[r])[pos]
        e = max(float(np.max(np.abs(o - go))), float(np.max(np.abs(lse - gl))))
        worst = max(worst, e)
    assert worst <= TOL[dtype], f"sampled per-round max-abs error {worst:.3e}"
    return worst
