"""Pins of the index-preparation and top-k-transform oracle (CPU).

Each expectation below is built independently of the oracle's loops:
slicing and concatenation for the ragged buffer (the construction the
review on the "reuse inference metadata and streamline FP8 prefill" page
asks for, HOLD rows included), cumulative sums for the ranges, the identity
page table of the "bench_mqa_logits_chunking.py" page (`_build`:
``page_table_1 = arange(n)``), and the paged oracle's own logits for the
64-token block table.
"""
import numpy as np
import pytest

import oracle
from oracle import index_prep as ip
from fp8_mqa_logits_03_b200 import workloads


def _table(rows, ld, seed):
    g = np.random.default_rng(seed)
    return g.integers(0, 1 << 30, size=(rows, ld)).astype(np.int32)


def test_ragged_buffer_matches_the_reviews_expected_layout():
    """One long request at table row 2, one of 4096 tokens at row 0, and four
    HOLD padding requests of 2 tokens that all name the HOLD row."""
    context_length, hold = 40000, 5
    table = _table(8, context_length + 16, 1)
    seq = [context_length, 4096, 2, 2, 2, 2]
    req = [2, 0, hold, hold, hold, hold]
    q = [1] * len(seq)
    capacity = context_length + 4096 + 8 + 37
    ks, ke, rt, ragged, tq, tk = ip.prepare_ragged(seq, q, req, table, q_cap=len(seq), ragged_cap=capacity)
    expected = np.full(capacity, -1, np.int32)
    expected[:context_length] = table[2, :context_length]
    expected[context_length:context_length + 4096] = table[0, :4096]
    expected[context_length + 4096:context_length + 4096 + 8] = np.tile(table[hold, :2], 4)
    assert np.array_equal(ragged, expected)
    assert tk == context_length + 4096 + 8 and tq == len(seq)


@pytest.mark.parametrize("q_len", [1, 4, 16])
def test_ranges_are_causal_tails_of_each_segment(q_len):
    g = np.random.default_rng(q_len)
    seq = g.integers(q_len, 3000, size=7).tolist()
    seq[3] = q_len                       # a request that is all query
    table = _table(9, 3000, 2)
    req = g.integers(0, 9, size=7).tolist()
    q = [q_len] * 7
    ks, ke, rt, _, tq, _ = ip.prepare_ragged(seq, q, req, table, q_cap=7 * q_len + 5)
    koff = np.concatenate([[0], np.cumsum(seq)])
    for b in range(7):
        rows = slice(b * q_len, (b + 1) * q_len)
        assert np.all(ks[rows] == koff[b])
        # the last row sees the whole request, each earlier row one key less
        assert np.array_equal(ke[rows] - ks[rows], np.arange(seq[b] - q_len + 1, seq[b] + 1))
        assert np.all(rt[rows] == req[b])
    assert np.all(ks[7 * q_len:] == 0) and np.all(ke[7 * q_len:] == 0) and np.all(rt[7 * q_len:] == -1)


def test_query_longer_than_sequence_clamps():
    ks, ke, _, _, _, _ = ip.prepare_ragged([3, 5], [5, 2], [0, 1], _table(2, 8, 3))
    assert ks.tolist() == [0, 0, 0, 0, 0, 3, 3]
    assert ke.tolist() == [0, 0, 1, 2, 3, 7, 8]


def test_transform_identity_table_gives_positions_within_the_request():
    """page_table_1 = arange(n) (one request, slot i = token i)."""
    n, rows, k = 5000, 6, 64
    g = np.random.default_rng(4)
    idx = g.integers(-1, n, size=(rows, k)).astype(np.int32)
    out = ip.topk_transform(idx, np.arange(n, dtype=np.int32)[None, :], 1, row_table=np.zeros(rows, np.int32))
    assert np.array_equal(out, np.where(idx >= 0, idx, -1))


def test_transform_through_ragged_layout_reaches_each_requests_own_slots():
    """A position j of row i in the ragged key space is token j - ks[i] of the
    row's request: the transform equals the ragged buffer at j."""
    seq, q = [700, 1300, 64], [4, 4, 4]
    table = _table(3, 1400, 5)
    req = [1, 2, 0]
    ks, ke, rt, ragged, _, _ = ip.prepare_ragged(seq, q, req, table)
    g = np.random.default_rng(6)
    idx = np.stack([np.where(g.random(32) < 0.2, -1, g.integers(ks[i], ke[i], size=32))
                    for i in range(len(ks))]).astype(np.int32)
    out = ip.topk_transform(idx, table, 1, row_base=ks, row_table=rt)
    assert np.array_equal(out, np.where(idx >= 0, ragged[np.maximum(idx, 0)], -1))


def test_transform_block_table_selects_the_keys_the_paged_form_scores():
    """With page_size 64 and the block table, the slot of each logical
    position holds the key whose logit the paged oracle computes there."""
    d = workloads.make_paged(3, 4, 100, 700, seed=9, lengths=[130, 700, 64])
    D = workloads.D
    R = 4
    rows = np.arange(3 * R)
    pos = np.stack([np.arange(0, 64) % max(1, int(d["seq_lens"][r // R])) for r in rows]).astype(np.int32)
    slots = ip.topk_transform(pos, d["block_table"].numpy(), 64, rows_per_table_row=R)
    ref = oracle.paged_logits_rows(d["q"].numpy(), d["k_pages"].numpy(), d["s_pages"].numpy(),
                                   d["w"].numpy(), d["block_table"].numpy(), d["seq_lens"].numpy(), R,
                                   rows=rows)
    kflat = d["k_pages"].numpy().reshape(-1, D)
    sflat = d["s_pages"].numpy().reshape(-1)
    for r in rows:
        keys, scales = kflat[slots[r]], sflat[slots[r]]
        direct = oracle.mqa_logits_rows(d["q"].numpy()[r:r + 1], keys, scales, d["w"].numpy()[r:r + 1],
                                        np.zeros(1, np.int32), np.full(1, 64, np.int32))[0]
        want = ref[r - rows[0], pos[r]]
        live = np.isfinite(want)
        assert np.allclose(direct[live], want[live], rtol=0, atol=0)


def test_transform_out_of_table_positions_map_to_minus_one():
    table = np.array([[3, -1, 7], [1, 2, 0]], np.int32)
    idx = np.array([[0, 63, 64, 130, 191, 192, -1, 5]], np.int32)
    out = ip.topk_transform(idx, table, 64, row_table=np.array([0], np.int32))
    assert out.tolist() == [[3 * 64, 3 * 64 + 63, -1, 7 * 64 + 2, 7 * 64 + 63, -1, -1, 3 * 64 + 5]]
    out = ip.topk_transform(idx, table, 64, row_table=np.array([2], np.int32))
    assert np.all(out == -1)
