"""Failure reporting through the device status word (needs a B200).

Every failure here is made on the host, in a form the library's own checks
turn into a status bit; nothing faults, traps or waits without a limit:

* a key-tile load the producer never issues (the library's test hook) with
  a 2 ms wait limit: the MMA's wait on that tile runs out, the kernel flags
  WAIT_TIMEOUT, every role leaves, drains its own copies and MMAs, frees its
  tensor memory and returns;
* a block-table entry outside the page pool: the producer skips that page's
  load and the scale read returns 0, flagging BAD_PAGE;
* a context length beyond max_blocks * 64: the request is clamped to the
  block table, flagging SEQ_TOO_LONG.

After each, a call with valid inputs and the default limit is clean and
matches the oracle, so the context stays usable.
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_mqa_logits_03_b200 as fx
from fp8_mqa_logits_03_b200 import workloads
from _parity import check_topk_row, row_range, paged_range

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_NS = 2_000_000_000


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp8_mqa_logits_03_b200 import build
    build.build()
    fx.lib()
    yield
    fx.set_wait_limit_ns(DEFAULT_LIMIT_NS)
    fx.debug_withhold_first_tile(False)


def _prefill(m, n, seed):
    d = workloads.make_prefill(m, n, seed)
    t = {k: d[k].cuda() for k in ("q", "k", "s", "w", "ks", "ke")}
    return d, t


def _check_prefill(d, idx, k):
    ref = oracle.mqa_logits_rows(d["q"].numpy(), d["k"].numpy(), d["s"].numpy(), d["w"].numpy(),
                                 d["ks"].numpy(), d["ke"].numpy(), rows=np.arange(d["m"]))
    for i in range(d["m"]):
        lo, hi = row_range(d["ks"][i], d["ke"][i], d["n"])
        check_topk_row(idx[i], ref[i], lo, hi, k, what=f"row {i}")


@pytest.mark.parametrize("m,n", [(16, 4096), (8 * 148, 3000)])  # split schedule + merge; direct
def test_wait_timeout_sets_status_and_recovers(m, n):
    d, t = _prefill(m, n, 61)
    ws = fx.alloc_workspace(fx.mqa_logits_topk_workspace_size(m, n, 512))
    try:
        fx.set_wait_limit_ns(2_000_000)
        fx.debug_withhold_first_tile(True)
        fx.mqa_logits_topk(**t, topk=512, workspace=ws)
        st = fx.read_device_status(ws)
    finally:
        fx.debug_withhold_first_tile(False)
        fx.set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert st & fx.STATUS_WAIT_TIMEOUT, f"status {st:#x}"
    idx = fx.mqa_logits_topk(**t, topk=512, workspace=ws)
    assert fx.read_device_status(ws) == 0
    if m <= 16:
        _check_prefill(d, idx.cpu().numpy(), 512)


def _paged(lengths, R=4, seed=62, max_blocks=None):
    d = workloads.make_paged(len(lengths), R, 1, max(lengths), seed=seed, lengths=lengths,
                             max_blocks=max_blocks)
    t = {k: d[k].cuda() for k in ("q", "k_pages", "s_pages", "w", "block_table", "seq_lens")}
    return d, t


def _run_paged(d, t, k=256):
    ws = fx.alloc_workspace(fx.paged_workspace_size(d["B"], d["R"], t["block_table"].shape[1], k))
    idx = fx.paged_mqa_logits_topk(**t, R=d["R"], topk=k, workspace=ws)
    return idx, fx.read_device_status(ws)


def test_paged_wait_timeout_sets_status_and_recovers():
    d, t = _paged([3000, 700, 1500, 64])
    try:
        fx.set_wait_limit_ns(2_000_000)
        fx.debug_withhold_first_tile(True)
        _, st = _run_paged(d, t)
    finally:
        fx.debug_withhold_first_tile(False)
        fx.set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert st & fx.STATUS_WAIT_TIMEOUT, f"status {st:#x}"
    _, st = _run_paged(d, t)
    assert st == 0


def test_bad_page_sets_status():
    d, t = _paged([3000, 700, 1500])
    bt = t["block_table"].clone()
    bt[1, 3] = d["P"] + 5        # past the pool
    bt[2, 0] = d["P"]            # just past the pool
    t_bad = dict(t, block_table=bt)
    _, st = _run_paged(d, t_bad)
    assert st & fx.STATUS_BAD_PAGE, f"status {st:#x}"
    idx, st = _run_paged(d, t)   # the same pool with a valid table is clean
    assert st == 0
    rows = np.arange(d["B"] * d["R"])
    ref = oracle.paged_logits_rows(d["q"].numpy(), d["k_pages"].numpy(), d["s_pages"].numpy(),
                                   d["w"].numpy(), d["block_table"].numpy(), d["seq_lens"].numpy(),
                                   d["R"], rows=rows)
    idx = idx.cpu().numpy()
    for r in rows:
        lo, hi = paged_range(int(d["seq_lens"][r // d["R"]]), d["R"], r % d["R"])
        check_topk_row(idx[r], ref[r], lo, hi, 256, what=f"row {r}")


def test_seq_len_beyond_block_table_sets_status():
    d, t = _paged([2000, 640], max_blocks=32)     # 32 blocks hold 2048 tokens
    sl = t["seq_lens"].clone()
    sl[0] = 32 * 64 + 100
    _, st = _run_paged(d, dict(t, seq_lens=sl))
    assert st & fx.STATUS_SEQ_TOO_LONG, f"status {st:#x}"
    _, st = _run_paged(d, t)
    assert st == 0
