"""The allocation-free fused entry point against the workspace one (needs a B200).

Some callers cannot allocate device memory at the moment they call the
indexer: code running under a CUDA graph that a framework captured and owns,
or a serving runtime whose memory budget is fixed at start-up.  For them the
library exposes fp8idx_mqa_logits_topk_noalloc, which takes its scratch from a
fixed device array inside the library instead of a caller workspace.  This
file calls it through the C ABI twice in a row (the array keeps the previous
call's contents) and checks each result against fp8idx_mqa_logits_topk on the
same inputs, reading the call's device status through the same ABI
(FP8IDX_NOALLOC_WS); one shape is also checked against the float64 oracle
directly.  It is collected last so that a run stopping at the first failure
has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import fp8_mqa_logits_03_b200 as fx
from fp8_mqa_logits_03_b200 import workloads
from _parity import check_topk_row, row_range

pytestmark = pytest.mark.gpu

ATOL = 1e-3
RTOL = 1e-3


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp8_mqa_logits_03_b200 import build
    build.build()
    lib = fx.lib()
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.fp8idx_mqa_logits_topk_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i32, i32, i32,
                                                   vp, vp, vp]
    lib.fp8idx_mqa_logits_topk_noalloc.restype = ctypes.c_int
    return lib


NOALLOC_WS = ctypes.c_void_p(1)  # FP8IDX_NOALLOC_WS


def _noalloc_status(L, stream):
    v = ctypes.c_int(-1)
    assert L.fp8idx_read_device_status(NOALLOC_WS, ctypes.byref(v), stream) == 0, L.fp8idx_last_error()
    return v.value


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _same_topk(got_i, got_v, ref_i, ref_v, k, what):
    """Equal index sets, except keys whose logit lies within the tolerance of
    the reference row's k-th value; values equal within the tolerance."""
    g = {int(j): float(v) for j, v in zip(got_i, got_v) if j >= 0}
    r = {int(j): float(v) for j, v in zip(ref_i, ref_v) if j >= 0}
    assert len(g) == len(r), what
    if not r:
        return
    T = min(r.values())
    tol = ATOL + RTOL * abs(T)
    for j in set(g) ^ set(r):
        v = g.get(j, r.get(j))
        assert abs(v - T) <= tol, f"{what}: key {j} ({v}) outside the tie band of {T}"
    for j in set(g) & set(r):
        assert abs(g[j] - r[j]) <= ATOL + RTOL * abs(r[j]), what


@pytest.mark.parametrize("m,n,k,seed", [
    (40, 6000, 512, 7),        # ragged rows, split key axis
    (16, 4096, 2048, 8),       # the tiny workload's shape
    (1200, 3000, 2048, 9),     # one unit per row block
    (8192, 35000, 2048, 10),   # the causal-prefill shape: the grid shrinks to fit the scratch
])
def test_noalloc_matches_workspace_entry_point_twice(L, m, n, k, seed):
    d = workloads.make_prefill(m, n, seed)
    t = {x: d[x].cuda() for x in ("q", "k", "s", "w", "ks", "ke")}
    ref_i, ref_v = fx.mqa_logits_topk(**t, topk=k, return_values=True)
    ref_i, ref_v = ref_i.cpu().numpy(), ref_v.cpu().numpy()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full((m, k), -7, dtype=torch.int32, device="cuda")
        vals = torch.full((m, k), 7.0, dtype=torch.float32, device="cuda")
        rc = L.fp8idx_mqa_logits_topk_noalloc(_p(t["q"]), _p(t["k"]), _p(t["s"]), _p(t["w"]),
                                              _p(t["ks"]), _p(t["ke"]), m, n, 32, 128, k, _p(out),
                                              _p(vals), stream)
        assert rc == 0, L.fp8idx_last_error()
        assert _noalloc_status(L, stream) == 0
        oi, ov = out.cpu().numpy(), vals.cpu().numpy()
        rows = range(m) if m <= 1200 else np.linspace(0, m - 1, 200).astype(int)
        for i in rows:
            _same_topk(oi[i], ov[i], ref_i[i], ref_v[i], k, f"call {call} row {i}")


def test_noalloc_matches_oracle(L):
    m, n, k = 24, 5000, 512
    g = np.random.default_rng(12)
    ks = g.integers(0, 200, size=m).astype(np.int32)
    ke = (ks + g.integers(100, n, size=m)).astype(np.int32)
    d = workloads.make_prefill(m, n, 12, ks=ks, ke=ke)
    t = {x: d[x].cuda() for x in ("q", "k", "s", "w", "ks", "ke")}
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    out = torch.empty((m, k), dtype=torch.int32, device="cuda")
    vals = torch.empty((m, k), dtype=torch.float32, device="cuda")
    rc = L.fp8idx_mqa_logits_topk_noalloc(_p(t["q"]), _p(t["k"]), _p(t["s"]), _p(t["w"]), _p(t["ks"]),
                                          _p(t["ke"]), m, n, 32, 128, k, _p(out), _p(vals), stream)
    assert rc == 0, L.fp8idx_last_error()
    assert _noalloc_status(L, stream) == 0
    ref = oracle.mqa_logits_rows(d["q"].numpy(), d["k"].numpy(), d["s"].numpy(), d["w"].numpy(),
                                 d["ks"].numpy(), d["ke"].numpy(), rows=np.arange(m))
    oi, ov = out.cpu().numpy(), vals.cpu().numpy()
    for i in range(m):
        lo, hi = row_range(d["ks"][i], d["ke"][i], n)
        check_topk_row(oi[i], ref[i], lo, hi, k, ov[i], f"row {i}")


def test_noalloc_rejects_bad_arguments(L):
    fake = ctypes.c_void_p(4096)
    assert L.fp8idx_mqa_logits_topk_noalloc(fake, fake, fake, fake, fake, fake, 4, 10, 16, 128, 8,
                                            fake, None, None) == fx.EUNSUPPORTED
    assert L.fp8idx_mqa_logits_topk_noalloc(fake, fake, fake, fake, fake, fake, 4, 10, 32, 128, 0,
                                            fake, None, None) == fx.EINVAL
