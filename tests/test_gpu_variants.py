"""Variants of the indexer against the oracle (needs a B200): MTP verify
widths 1..8 rows per request in the paged form (the megakernels page names
uniform q4-q8 verify metadata; 1 is plain decode) and 64 index heads in the
prefill, logits and paged forms."""
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


def _paged(lengths, R, k, seed, heads=workloads.H):
    d = workloads.make_paged(len(lengths), R, 1, max(lengths), seed=seed, lengths=lengths, heads=heads)
    t = {x: d[x].cuda() for x in ("q", "k_pages", "s_pages", "w", "block_table", "seq_lens")}
    ws = fx.alloc_workspace(fx.paged_workspace_size(len(lengths), R, d["max_blocks"], k, heads))
    idx, vals = fx.paged_mqa_logits_topk(**t, R=R, topk=k, return_values=True, workspace=ws)
    assert fx.read_device_status(ws) == 0
    rows = np.arange(len(lengths) * R)
    ref = oracle.paged_logits_rows(d["q"].numpy(), d["k_pages"].numpy(), d["s_pages"].numpy(),
                                   d["w"].numpy(), d["block_table"].numpy(), d["seq_lens"].numpy(), R,
                                   rows=rows)
    idx, vals = idx.cpu().numpy(), vals.cpu().numpy()
    for r in rows:
        lo, hi = paged_range(int(d["seq_lens"][r // R]), R, r % R)
        check_topk_row(idx[r], ref[r], lo, hi, k, vals[r], f"R={R} row {r}")


@pytest.mark.parametrize("R", [1, 2, 3, 5, 6, 7])
def test_paged_mtp_widths(R):
    lengths = [1, 5, 64, 130, 3000, 5000, 2049, 700]
    _paged(lengths, R, 512 if R % 2 else 2048, seed=70 + R)


def _prefill64(m, n, k, seed, ragged=True):
    if ragged:
        g = np.random.default_rng(seed)
        ks = g.integers(-5, n // 3, size=m).astype(np.int32)
        ke = (ks + g.integers(0, n, size=m)).astype(np.int32)
        d = workloads.make_prefill(m, n, seed, ks=ks, ke=ke, heads=64)
    else:
        d = workloads.make_prefill(m, n, seed, heads=64)
    return d, {x: d[x].cuda() for x in ("q", "k", "s", "w", "ks", "ke")}


@pytest.mark.parametrize("m,n,k", [(13, 6000, 512), (4 * 148 + 3, 3000, 2048)])  # split + merge; direct
def test_fused_64_heads(m, n, k):
    d, t = _prefill64(m, n, k, 80 + m)
    idx, vals = fx.mqa_logits_topk(**t, topk=k, return_values=True)
    rows = np.arange(m) if m < 64 else np.concatenate([np.arange(0, 12), np.arange(m - 12, m)])
    ref = oracle.mqa_logits_rows(d["q"].numpy(), d["k"].numpy(), d["s"].numpy(), d["w"].numpy(),
                                 d["ks"].numpy(), d["ke"].numpy(), rows=rows)
    idx, vals = idx.cpu().numpy(), vals.cpu().numpy()
    for r, i in enumerate(rows):
        lo, hi = row_range(d["ks"][i], d["ke"][i], n)
        check_topk_row(idx[i], ref[r], lo, hi, k, vals[i], f"row {i}")


def test_logits_64_heads():
    m, n = 9, 2000
    d, t = _prefill64(m, n, 0, 90)
    lg = fx.mqa_logits(**t)
    torch.cuda.synchronize()
    check_logits(lg.cpu().numpy(), oracle.mqa_logits_rows(d["q"].numpy(), d["k"].numpy(), d["s"].numpy(),
                                                          d["w"].numpy(), d["ks"].numpy(), d["ke"].numpy()))


@pytest.mark.parametrize("R", [1, 4])
def test_paged_64_heads(R):
    _paged([3000, 64, 5000, 129], R, 512, seed=95 + R, heads=64)


def test_unsupported_shapes_are_rejected():
    d = workloads.make_paged(2, 5, 1, 200, seed=1, lengths=[100, 200], heads=64)
    t = {x: d[x].cuda() for x in ("q", "k_pages", "s_pages", "w", "block_table", "seq_lens")}
    with pytest.raises(fx.Fp8IdxError) as e:
        fx.paged_mqa_logits_topk(**t, R=5, topk=16, workspace=fx.alloc_workspace(1 << 20))
    assert e.value.code == fx.EUNSUPPORTED
