"""Comparison rules between the CUDA path and the float64 oracle.

Logits: |gpu - oracle| <= 1e-3 + 1e-3 * |oracle| on valid entries, and -inf
exactly where the oracle has -inf.

Top-k (per row): no duplicates; every index inside the row's valid range;
exactly min(k, valid) indices followed by -1 padding; when valid <= k the
set is all valid keys; otherwise every key in the symmetric difference of
the GPU set and the oracle set has an oracle logit within the same
tolerance of the oracle's k-th value T.
"""
from __future__ import annotations

import numpy as np

ATOL = 1e-3
RTOL = 1e-3


def check_logits(gpu: np.ndarray, ref: np.ndarray, what: str = "logits"):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    ninf = np.isneginf(ref)
    bad_inf = np.isneginf(gpu) != ninf
    assert not bad_inf.any(), f"{what}: -inf mismatch at {np.argwhere(bad_inf)[:5].tolist()}"
    fin = ~ninf
    err = np.abs(gpu[fin] - ref[fin])
    lim = ATOL + RTOL * np.abs(ref[fin])
    if err.size:
        worst = int(np.argmax(err - lim))
        assert np.all(err <= lim), (f"{what}: max excess {float((err - lim)[worst]):.3g} "
                                    f"(gpu {gpu[fin][worst]}, ref {ref[fin][worst]})")
    return float(err.max()) if err.size else 0.0


def check_topk_row(gpu_idx: np.ndarray, ref_row: np.ndarray, lo: int, hi: int, k: int,
                   gpu_vals: np.ndarray | None = None, what: str = "row"):
    """gpu_idx [k] int32 from the kernel; ref_row: the oracle's float64 logits of
    the row over the whole key axis (-inf outside [lo, hi))."""
    gpu_idx = np.asarray(gpu_idx)
    cnt = max(0, hi - lo)
    want = min(k, cnt)
    nvalid = int((gpu_idx >= 0).sum())
    assert nvalid == want, f"{what}: {nvalid} indices, expected {want}"
    assert np.all(gpu_idx[:want] >= 0) and np.all(gpu_idx[want:] == -1), f"{what}: padding not at tail"
    sel = gpu_idx[:want].astype(np.int64)
    assert len(np.unique(sel)) == want, f"{what}: duplicate indices"
    assert np.all((sel >= lo) & (sel < hi)), f"{what}: index outside [{lo}, {hi})"
    if gpu_vals is not None:
        check_logits(np.asarray(gpu_vals)[:want], ref_row[sel], what + " values")
        assert np.all(np.isneginf(np.asarray(gpu_vals)[want:])), f"{what}: value padding"
    if cnt <= k:
        assert set(sel.tolist()) == set(range(lo, hi)), f"{what}: short row must select all"
        return 0
    seg = ref_row[lo:hi]
    order = np.lexsort((np.arange(lo, hi), -seg))  # value desc, index asc
    ref_set = set((order[:k] + lo).tolist())
    T = seg[order[k - 1]]
    diff = ref_set.symmetric_difference(sel.tolist())
    tol = ATOL + RTOL * abs(T)
    for j in diff:
        assert abs(ref_row[j] - T) <= tol, (f"{what}: key {j} (oracle {ref_row[j]}) differs from the "
                                            f"oracle set outside the tie band around T={T}")
    return len(diff)


def row_range(ks: int, ke: int, n: int):
    lo = max(int(ks), 0)
    hi = max(lo, min(int(ke), n))
    return lo, hi


def paged_range(L: int, R: int, t: int):
    e = L - R + t + 1
    return 0, max(0, min(e, L))
