"""Index preparation and the top-k transform, written out plainly -- TEST
INFRASTRUCTURE ONLY (same rule as the rest of ``oracle/``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s reference legs use it).

What is computed follows the "reuse inference metadata and streamline FP8
prefill" page (LightLLM pull request: its description table, the
``gen_nsa_ks_ke`` walkthrough and the review's expected ragged buffer) and
the ``page_table_size_1`` argument of ``fast_topk_transform_fused`` on the
"bench_mqa_logits_chunking.py" page (``_build``, ``_run_chunked``):

* Requests b = 0..B-1 are laid out back to back in one "ragged" key space:
  request b owns key positions [koff_b, koff_b + seq_len[b]) with
  koff_b = sum of the earlier seq_len.  Its query rows (its last q_len[b]
  tokens) are also back to back, from qoff_b = sum of the earlier q_len.
* Query row t of request b sees its request's causal prefix:
      ks = koff_b,  ke = koff_b + clamp(seq_len[b] - q_len[b] + t + 1, 0, seq_len[b]).
* The ragged index buffer holds every request's token slots in that order:
      ragged[koff_b + p] = req_to_token[req_idx[b], p]   for p < seq_len[b]
  (the review's expected buffer is exactly this concatenation; several batch
  entries may name the same table row, as the HOLD padding requests do).
* The top-k transform maps a selected position to a physical slot through a
  page table of `page_size`-token pages (page_size 1: a token-granular table
  such as ``page_table_size_1`` or ``req_to_token``):
      p = idx - base_row,  slot = table[trow, p // page_size] * page_size + p % page_size,
  and -1 stays -1; a position or page outside the table maps to -1.

Pure-Python loops: meant for the small cases the tests use.
"""
from __future__ import annotations

import numpy as np


def prepare_ragged(seq_len, q_len, req_idx, req_to_token, q_cap: int | None = None,
                   ragged_cap: int | None = None):
    """Returns (ks, ke, row_table, ragged, total_q, total_k).  Rows past the
    batch's rows up to q_cap are empty (ks = ke = 0, row_table = -1); the
    ragged buffer past total_k up to ragged_cap is -1 (untouched)."""
    seq_len = [int(x) for x in seq_len]
    q_len = [int(x) for x in q_len]
    req_idx = [int(x) for x in req_idx]
    table = np.asarray(req_to_token)
    ks, ke, row_table, ragged = [], [], [], []
    koff = 0
    for b in range(len(seq_len)):
        L, Q = seq_len[b], q_len[b]
        for t in range(Q):
            ks.append(koff)
            ke.append(koff + min(max(L - Q + t + 1, 0), L))
            row_table.append(req_idx[b])
        for p in range(L):
            ragged.append(int(table[req_idx[b], p]))
        koff += L
    total_q, total_k = len(ks), len(ragged)
    q_cap = total_q if q_cap is None else q_cap
    ragged_cap = total_k if ragged_cap is None else ragged_cap
    out_ks = np.zeros(q_cap, np.int32)
    out_ke = np.zeros(q_cap, np.int32)
    out_rt = np.full(q_cap, -1, np.int32)
    out_rg = np.full(ragged_cap, -1, np.int32)
    nq, nk = min(total_q, q_cap), min(total_k, ragged_cap)
    out_ks[:nq] = ks[:nq]
    out_ke[:nq] = ke[:nq]
    out_rt[:nq] = row_table[:nq]
    out_rg[:nk] = ragged[:nk]
    return out_ks, out_ke, out_rt, out_rg, total_q, total_k


def topk_transform(idx, page_table, page_size: int, row_base=None, row_table=None,
                   rows_per_table_row: int = 1):
    """out[i, r] = slot of position idx[i, r] - row_base[i] in table row
    row_table[i] (or i // rows_per_table_row); -1 where idx is -1 or the
    position / page falls outside the table."""
    idx = np.asarray(idx)
    table = np.asarray(page_table)
    rows, k = idx.shape
    n_trows, ld = table.shape
    out = np.full((rows, k), -1, np.int32)
    for i in range(rows):
        base = 0 if row_base is None else int(row_base[i])
        trow = int(row_table[i]) if row_table is not None else i // rows_per_table_row
        if not 0 <= trow < n_trows:
            continue
        for r in range(k):
            v = int(idx[i, r])
            if v < 0:
                continue
            p = v - base
            if p < 0 or p // page_size >= ld:
                continue
            page = int(table[trow, p // page_size])
            if page < 0:
                continue
            out[i, r] = page * page_size + p % page_size
    return out
