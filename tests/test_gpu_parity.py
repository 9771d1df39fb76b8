"""CUDA path vs the float64 oracle, element by element (needs a B200).

Small shapes span several 128-key tiles with a ragged tail, several 8-row
blocks with a partial last block, ragged/empty/clamped ranges, and both the
direct (one key chunk per row block) and the split (key chunks + merge)
schedules.  The full-size workloads are checked on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_mqa_logits_03_b200 as fx
from fp8_mqa_logits_03_b200 import workloads
from _parity import check_logits, check_topk_row, row_range, paged_range

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp8_mqa_logits_03_b200 import build
    build.build()
    fx.lib()


def _to(d, keys=("q", "k", "s", "w", "ks", "ke")):
    return {k: d[k].cuda() for k in keys}


def _ragged(m, n, seed):
    g = np.random.default_rng(seed)
    ks = g.integers(-20, n // 2, size=m).astype(np.int32)
    ke = (ks + g.integers(-5, n, size=m)).astype(np.int32)
    ke[0], ks[0] = n + 50, -3          # clamped on both sides
    ks[1], ke[1] = 7, 7                # empty
    ks[2], ke[2] = 40, 10              # reversed = empty
    if m > 3:
        ks[3], ke[3] = n - 1, n        # a single key
    return ks, ke


def _oracle_rows(d, rows):
    return oracle.mqa_logits_rows(d["q"].numpy(), d["k"].numpy(), d["s"].numpy(), d["w"].numpy(),
                                  d["ks"].numpy(), d["ke"].numpy(), rows=np.asarray(rows))


# ---------------------------------------------------------------------------- logits

@pytest.mark.parametrize("m,n,seed", [(20, 1000, 1), (16, 4096, 2), (3, 129, 3), (1, 1, 4)])
def test_mqa_logits_small(m, n, seed):
    ks, ke = _ragged(m, n, seed) if m >= 4 else (np.zeros(m, np.int32), np.full(m, n, np.int32))
    d = workloads.make_prefill(m, n, seed, ks=ks, ke=ke)
    t = _to(d)
    lg = fx.mqa_logits(**t)
    torch.cuda.synchronize()
    ref = _oracle_rows(d, np.arange(m))
    check_logits(lg.cpu().numpy(), ref)


def test_mqa_logits_many_row_blocks_strided_output():
    """Enough rows for the unsplit schedule (>= 8 x SMs); output with ld > n."""
    m, n = 8 * fx.num_sms() + 13, 700
    d = workloads.make_prefill(m, n, 11)
    t = _to(d)
    out = torch.full((m, n + 37), 7.0, device="cuda")
    fx.mqa_logits(**t, logits=out[:, :n])
    torch.cuda.synchronize()
    rows = np.concatenate([np.arange(0, 9), np.arange(m - 9, m), np.arange(500, 520)])
    ref = _oracle_rows(d, rows)
    check_logits(out[rows, :n].cpu().numpy(), ref)
    assert torch.all(out[:, n:] == 7.0)  # nothing written past n


# ---------------------------------------------------------------------------- top-k of rows

@pytest.mark.parametrize("m,n,k", [(7, 5000, 2048), (5, 300, 2048), (33, 3000, 64), (4, 70000, 2048)])
def test_topk_rows_exact(m, n, k):
    g = torch.Generator().manual_seed(m * 1000 + n)
    lg = (torch.randn(m, n, generator=g) * 8).round() / 4  # many exact ties
    ks, ke = _ragged(m, n, n)
    gpu = fx.topk_rows(lg.cuda(), torch.from_numpy(ks).cuda(), torch.from_numpy(ke).cuda(), k)
    torch.cuda.synchronize()
    ref_idx, _ = oracle.topk_rows(lg.double().numpy(), ks, ke, k)
    gpu = gpu.cpu().numpy()
    for i in range(m):
        want = ref_idx[i]
        assert sorted(gpu[i][gpu[i] >= 0].tolist()) == sorted(want[want >= 0].tolist()), i
        assert np.all(gpu[i][(want >= 0).sum():] == -1)


# ---------------------------------------------------------------------------- fused

def _fused_call(d, k, values=True):
    """Fused call with an explicit workspace; asserts the device status is clean."""
    t = _to(d)
    ws = fx.alloc_workspace(fx.mqa_logits_topk_workspace_size(d["m"], d["n"], k))
    out = fx.mqa_logits_topk(**t, topk=k, return_values=values, workspace=ws)
    assert fx.read_device_status(ws) == 0
    return out


def _check_fused(d, idx, vals, rows, k):
    ref = _oracle_rows(d, rows)
    n = d["n"]
    for r, i in enumerate(rows):
        lo, hi = row_range(d["ks"][i], d["ke"][i], n)
        check_topk_row(idx[i], ref[r], lo, hi, k, None if vals is None else vals[i], f"row {i}")


@pytest.mark.parametrize("m,n,k,seed", [
    (20, 1000, 2048, 1),     # split schedule, rows shorter than k
    (16, 4096, 2048, 2),     # the tiny workload's shape
    (13, 9000, 2048, 3),     # split schedule, rows longer than k
    (9, 6000, 64, 4),        # small k: many in-kernel compactions
    (11, 7000, 512, 5),      # top-512, the GLM-5.3-Flash indexer width
    (10, 3000, 1, 6),        # k = 1: an argmax per row (lowest index on ties)
    (10, 5000, 2047, 7),     # k just below the maximum, odd
])
def test_fused_small(m, n, k, seed):
    ks, ke = _ragged(m, n, seed)
    d = workloads.make_prefill(m, n, seed, ks=ks, ke=ke)
    idx, vals = _fused_call(d, k)
    _check_fused(d, idx.cpu().numpy(), vals.cpu().numpy(), np.arange(m), k)


@pytest.mark.parametrize("m,n,k,seed", [(13, 9000, 2048, 41), (8 * 148 + 3, 5000, 512, 42)])
def test_fused_signed_weights(m, n, k, seed):
    """Head weights of both signs, w ~ U[-1, 1): heads cancel in the weighted sum,
    which is where the epilogue's w*x + w*|x| form and the plain ReLU form differ most."""
    ks, ke = _ragged(m, n, seed)
    d = workloads.make_prefill(m, n, seed, ks=ks, ke=ke, signed_weights=True)
    idx, vals = _fused_call(d, k)
    rows = np.arange(m) if m < 64 else np.concatenate([np.arange(0, 16), np.arange(m - 16, m)])
    _check_fused(d, idx.cpu().numpy(), vals.cpu().numpy(), rows, k)


def test_mqa_logits_signed_weights():
    m, n = 24, 3000
    ks, ke = _ragged(m, n, 43)
    d = workloads.make_prefill(m, n, 43, ks=ks, ke=ke, signed_weights=True)
    lg = fx.mqa_logits(**_to(d))
    torch.cuda.synchronize()
    check_logits(lg.cpu().numpy(), _oracle_rows(d, np.arange(m)))


@pytest.mark.parametrize("k", [2048, 100])
def test_fused_unsplit_schedule(k):
    """>= 8 x SMs rows: one unit per row block, top-k written directly."""
    m, n = 8 * fx.num_sms() + 5, 5000 if k == 2048 else 2500
    d = workloads.make_prefill(m, n, 21 + k)
    idx, vals = _fused_call(d, k)
    rows = np.concatenate([np.arange(0, 8), np.arange(m - 8, m), np.arange(400, 408)])
    _check_fused(d, idx.cpu().numpy(), vals.cpu().numpy(), rows, k)


def test_fused_equals_chained():
    """Fused and chained (mqa_logits -> topk_rows) paths agree on all rows."""
    m, n, k = 40, 6000, 512
    d = workloads.make_prefill(m, n, 31)
    t = _to(d)
    fused = fx.mqa_logits_topk(**t, topk=k)
    lg = fx.mqa_logits(**t)
    chained = fx.topk_rows(lg, t["ks"], t["ke"], k)
    torch.cuda.synchronize()
    f, c = fused.cpu().numpy(), chained.cpu().numpy()
    for i in range(m):
        assert sorted(f[i].tolist()) == sorted(c[i].tolist()), i


def test_fused_all_ties():
    """Every key identical: the top-k is the k lowest indices of each range."""
    m, n, k = 10, 3000, 256
    d = workloads.make_prefill(m, n, 5, duplicate_keys=True)
    idx = _fused_call(d, k, values=False).cpu().numpy()
    for i in range(m):
        lo, hi = row_range(d["ks"][i], d["ke"][i], n)
        want = list(range(lo, min(hi, lo + k)))
        assert sorted(idx[i][idx[i] >= 0].tolist()) == want, i


def test_fused_empty_inputs():
    d = workloads.make_prefill(5, 0, 1)
    t = {k: v.cuda() for k, v in d.items() if isinstance(v, torch.Tensor)}
    t["k"] = torch.empty((0, 128), dtype=torch.uint8, device="cuda")
    t["s"] = torch.empty((0,), dtype=torch.float32, device="cuda")
    idx, vals = fx.mqa_logits_topk(**t, topk=16, return_values=True)
    assert torch.all(idx == -1) and torch.all(torch.isneginf(vals))
    out = fx.mqa_logits_topk(t["q"][:0], t["k"], t["s"], t["w"][:0], t["ks"][:0], t["ke"][:0], topk=16)
    assert out.shape == (0, 16)


# ---------------------------------------------------------------------------- paged

def _paged_check(d, idx, vals, rows, k):
    ref = oracle.paged_logits_rows(d["q"].numpy(), d["k_pages"].numpy(), d["s_pages"].numpy(),
                                   d["w"].numpy(), d["block_table"].numpy(), d["seq_lens"].numpy(),
                                   d["R"], rows=np.asarray(rows))
    R = d["R"]
    for r, row in enumerate(rows):
        L = int(d["seq_lens"][row // R])
        lo, hi = paged_range(L, R, row % R)
        check_topk_row(idx[row], ref[r], lo, hi, k, None if vals is None else vals[row], f"row {row}")


@pytest.mark.parametrize("R,k", [(4, 2048), (8, 2048), (4, 100), (8, 512)])
def test_paged_small(R, k):
    lengths = [1, 3, 64, 65, 127, 128, 129, 700, 2100, 5000, 4097]
    d = workloads.make_paged(len(lengths), R, 1, 5000, seed=R + k, lengths=lengths)
    t = {key: d[key].cuda() for key in ("q", "k_pages", "s_pages", "w", "block_table", "seq_lens")}
    ws = fx.alloc_workspace(fx.paged_workspace_size(len(lengths), R, d["max_blocks"], k))
    idx, vals = fx.paged_mqa_logits_topk(**t, R=R, topk=k, return_values=True, workspace=ws)
    assert fx.read_device_status(ws) == 0
    _paged_check(d, idx.cpu().numpy(), vals.cpu().numpy(), np.arange(len(lengths) * R), k)


def test_paged_signed_weights():
    lengths = [5000, 300, 4200, 64, 2049, 9000]
    d = workloads.make_paged(len(lengths), 4, 1, 9000, seed=44, lengths=lengths, signed_weights=True)
    t = {key: d[key].cuda() for key in ("q", "k_pages", "s_pages", "w", "block_table", "seq_lens")}
    ws = fx.alloc_workspace(fx.paged_workspace_size(len(lengths), 4, d["max_blocks"], 2048))
    idx, vals = fx.paged_mqa_logits_topk(**t, R=4, topk=2048, return_values=True, workspace=ws)
    assert fx.read_device_status(ws) == 0
    _paged_check(d, idx.cpu().numpy(), vals.cpu().numpy(), np.arange(len(lengths) * 4), 2048)


# ---------------------------------------------------------------------------- full sizes (sampled)

def _sample_rows(m, count, seed):
    g = np.random.default_rng(seed)
    rows = set([0, 1, 7, 8, m - 1, m - 2, m - 8, m - 9])
    rows.update(g.choice(m, size=count, replace=False).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < m))


@pytest.mark.parametrize("index,count", [(0, 16), (1, 48), (2, 24), (3, 8)])
def test_fused_full_workloads_sampled(index, count):
    d = workloads.make_workload(index)
    idx, vals = _fused_call(d, workloads.TOPK)
    rows = _sample_rows(d["m"], min(count, d["m"]), index)
    _check_fused(d, idx.cpu().numpy(), vals.cpu().numpy(), rows, workloads.TOPK)


def test_paged_full_workload_sampled():
    d = workloads.make_workload(4)
    t = {key: d[key].cuda() for key in ("q", "k_pages", "s_pages", "w", "block_table", "seq_lens")}
    ws = fx.alloc_workspace(fx.paged_workspace_size(d["B"], d["R"], d["max_blocks"], workloads.TOPK))
    idx, vals = fx.paged_mqa_logits_topk(**t, R=d["R"], topk=workloads.TOPK, return_values=True,
                                         workspace=ws)
    assert fx.read_device_status(ws) == 0
    rows = _sample_rows(d["B"] * d["R"], 24, 4)
    _paged_check(d, idx.cpu().numpy(), vals.cpu().numpy(), rows, workloads.TOPK)


# ---------------------------------------------------------------------------- estimated thresholds

def _decaying_scales(n, rate):
    """Key scales that fall along the key axis: the first keys seen dominate,
    so a threshold estimated from them overshoots the row's k-th value."""
    return (1.5 * torch.exp(-rate * torch.arange(n, dtype=torch.float64))).to(torch.float32) + 1e-3


@pytest.mark.parametrize("m,n,k", [(40, 20000, 512), (6 * 148 + 3, 6000, 256)])  # split + merge; direct
def test_fused_estimate_rejected_and_repaired(m, n, k):
    """Adversarial key order: the estimate check rejects rows, their row blocks
    are recomputed exactly, and every row still matches the oracle."""
    d = workloads.make_prefill(m, n, 51)
    d["s"] = _decaying_scales(n, 6.0 / n)
    t = _to(d)
    ws = fx.alloc_workspace(fx.mqa_logits_topk_workspace_size(m, n, k))
    idx, vals = fx.mqa_logits_topk(**t, topk=k, return_values=True, workspace=ws)
    stats = fx.read_device_stats(ws)
    assert stats["status"] == 0
    assert stats["repairs"] > 0, stats
    rows = np.arange(m) if m <= 64 else np.concatenate([np.arange(0, 24), np.arange(m - 24, m)])
    _check_fused(d, idx.cpu().numpy(), vals.cpu().numpy(), rows, k)


def test_paged_estimate_rejected_and_repaired():
    lengths = [9000, 4000, 12000, 700]
    R, k = 4, 512
    d = workloads.make_paged(len(lengths), R, 1, 12000, seed=52, lengths=lengths)
    # scales falling with each request's logical position, written through its block table
    sp = d["s_pages"].clone().view(-1)
    for b, L in enumerate(lengths):
        pos = torch.arange(L)
        slots = d["block_table"][b, pos // 64].long() * 64 + pos % 64
        sp[slots] = _decaying_scales(L, 6.0 / L)
    d["s_pages"] = sp.view_as(d["s_pages"])
    t = {key: d[key].cuda() for key in ("q", "k_pages", "s_pages", "w", "block_table", "seq_lens")}
    ws = fx.alloc_workspace(fx.paged_workspace_size(len(lengths), R, d["max_blocks"], k))
    idx, vals = fx.paged_mqa_logits_topk(**t, R=R, topk=k, return_values=True, workspace=ws)
    stats = fx.read_device_stats(ws)
    assert stats["status"] == 0
    assert stats["repairs"] > 0, stats
    _paged_check(d, idx.cpu().numpy(), vals.cpu().numpy(), np.arange(len(lengths) * R), k)


# ---------------------------------------------------------------------------- wide samples, full rows

def _blocks_and_random(m, count, seed, block=8):
    """The first and last row blocks plus `count` random rows."""
    g = np.random.default_rng(seed)
    rows = set(range(min(block, m))) | set(range(max(0, m - block), m))
    rows.update(g.choice(m, size=min(count, m), replace=False).tolist())
    return np.array(sorted(rows))


def test_cp_slice_210k_fused_and_chained_sampled():
    """Workload 3 (7500 rows over 210000 keys): the fused call and the chained
    path (logits in row chunks of at most 2 GiB, then topk_rows on each chunk,
    the loop of the chunking benchmark) on the first and last row blocks and
    256 random rows, against one oracle evaluation."""
    d = workloads.make_workload(3)
    m, n, k = d["m"], d["n"], workloads.TOPK
    idx, vals = _fused_call(d, k)
    t = _to(d)
    rows_per_chunk = max(1, (2 << 30) // (4 * n))
    chained = torch.empty((m, k), dtype=torch.int32, device="cuda")
    logits = torch.empty((rows_per_chunk, n), dtype=torch.float32, device="cuda")
    for r0 in range(0, m, rows_per_chunk):
        r1 = min(m, r0 + rows_per_chunk)
        lg = logits[: r1 - r0]
        fx.mqa_logits(t["q"][r0:r1], t["k"], t["s"], t["w"][r0:r1], t["ks"][r0:r1], t["ke"][r0:r1], logits=lg)
        fx.topk_rows(lg, t["ks"][r0:r1], t["ke"][r0:r1], k, out=chained[r0:r1])
    torch.cuda.synchronize()
    assert fx.read_device_status(None) == 0
    rows = _blocks_and_random(m, 256, 3)
    ref = _oracle_rows(d, rows)
    fi, fv, ci = idx.cpu().numpy(), vals.cpu().numpy(), chained.cpu().numpy()
    for r, i in enumerate(rows):
        lo, hi = row_range(d["ks"][i], d["ke"][i], n)
        check_topk_row(fi[i], ref[r], lo, hi, k, fv[i], f"fused row {i}")
        check_topk_row(ci[i], ref[r], lo, hi, k, None, f"chained row {i}")


def test_causal_prefill_all_rows():
    """Workload 1 (8192 rows over 35000 keys), every row against the oracle."""
    d = workloads.make_workload(1)
    m, n, k = d["m"], d["n"], workloads.TOPK
    idx, vals = _fused_call(d, k)
    fi, fv = idx.cpu().numpy(), vals.cpu().numpy()
    diffs = 0
    for r0 in range(0, m, 512):
        rows = np.arange(r0, min(m, r0 + 512))
        ref = _oracle_rows(d, rows)
        for r, i in enumerate(rows):
            lo, hi = row_range(d["ks"][i], d["ke"][i], n)
            diffs += check_topk_row(fi[i], ref[r], lo, hi, k, fv[i], f"row {i}")
    print(f"all {m} rows match; {diffs} keys swapped inside the tie band")
