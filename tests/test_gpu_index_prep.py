"""Index preparation and the top-k transform on the GPU against the oracle,
bit for bit (needs a B200).  Integer work: every output must be identical."""
import numpy as np
import pytest
import torch

from oracle import index_prep as ip
from oracle import paged_logits_rows
import fp8_mqa_logits_03_b200 as fx
from fp8_mqa_logits_03_b200 import workloads
from _parity import check_topk_row, paged_range

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp8_mqa_logits_03_b200 import build
    build.build()
    fx.lib()


def _batch(B, max_len, q_choices, seed, table_rows=None, ld=None, hold=None):
    g = np.random.default_rng(seed)
    q = g.choice(q_choices, size=B).astype(np.int32)
    seq = np.maximum(g.integers(0, max_len, size=B), q).astype(np.int32)
    table_rows = table_rows or B + 3
    ld = ld or max_len + 5
    table = g.integers(0, 1 << 30, size=(table_rows, ld)).astype(np.int32)
    req = g.integers(0, table_rows, size=B).astype(np.int32)
    if hold is not None:                       # trailing HOLD padding requests
        req[-hold:] = table_rows - 1
        seq[-hold:] = 2
        q[-hold:] = 1
    return seq, q, req, table


def _gpu_prepare(seq, q, req, table, q_cap, ragged_cap):
    t = [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in (seq, q, req, table)]
    ragged = torch.full((ragged_cap,), -1, dtype=torch.int32, device="cuda")
    ks, ke, rt, rg = fx.prepare_ragged(*t, q_cap=q_cap, ragged=ragged)
    torch.cuda.synchronize()
    return ks.cpu().numpy(), ke.cpu().numpy(), rt.cpu().numpy(), rg.cpu().numpy()


@pytest.mark.parametrize("B,max_len,qc,seed,hold", [
    (1, 1, [1], 1, None),
    (8, 5000, [1], 2, None),            # decode
    (8, 5000, [4], 3, None),            # MTP-4 verify
    (13, 9000, [16], 4, None),          # 16 queries per request
    (40, 3000, [1, 4, 16], 5, 6),       # mixed widths, HOLD padding rows
    (600, 700, [1, 3], 6, 20),          # many requests (several scan passes per CTA)
])
def test_prepare_matches_oracle(B, max_len, qc, seed, hold):
    seq, q, req, table = _batch(B, max_len, qc, seed, hold=hold)
    tq, tk = int(q.sum()), int(seq.sum())
    for q_cap, ragged_cap in [(tq + 7, tk + 33), (tq, max(1, tk // 2))]:   # padded; truncated copy
        want = ip.prepare_ragged(seq, q, req, table, q_cap=q_cap, ragged_cap=ragged_cap)
        got = _gpu_prepare(seq, q, req, table, q_cap, ragged_cap)
        for name, a, b in zip(("ks", "ke", "row_table", "ragged"), got, want[:4]):
            assert np.array_equal(a, b), name


def test_prepare_long_context_layout():
    """The review's layout at 1M + 4096 tokens: the ragged buffer is the
    concatenation of the requests' table rows, HOLD rows included."""
    ctx, hold = 1 << 20, 7
    g = np.random.default_rng(11)
    table = g.integers(0, 1 << 30, size=(8, ctx + 64)).astype(np.int32)
    seq = np.array([ctx, 4096, 2, 2, 2, 2], np.int32)
    req = np.array([2, 0, hold, hold, hold, hold], np.int32)
    q = np.ones(6, np.int32)
    cap = ctx + 4096 + 8 + 100
    ks, ke, rt, rg = _gpu_prepare(seq, q, req, table, 6, cap)
    expected = np.full(cap, -1, np.int32)
    expected[:ctx] = table[2, :ctx]
    expected[ctx:ctx + 4096] = table[0, :4096]
    expected[ctx + 4096:ctx + 4096 + 8] = np.tile(table[hold, :2], 4)
    assert np.array_equal(rg, expected)
    koff = np.concatenate([[0], np.cumsum(seq)])
    assert np.array_equal(ks, koff[:6]) and np.array_equal(ke, koff[1:])


def test_transform_ragged_matches_oracle():
    seq, q, req, table = _batch(9, 4000, [1, 4, 16], 21, hold=2)
    ks, ke, rt, rg, tq, _ = ip.prepare_ragged(seq, q, req, table)
    g = np.random.default_rng(22)
    k = 256
    idx = np.stack([np.where(g.random(k) < 0.1, -1, g.integers(ks[i], max(ke[i], ks[i] + 1), size=k))
                    for i in range(tq)]).astype(np.int32)
    idx[0, :5] = [ks[0] - 1, ke[0] + 10 ** 6, -1, -5, ks[0]]      # out of the request, padding
    want = ip.topk_transform(idx, table, 1, row_base=ks, row_table=rt)
    t_idx = torch.from_numpy(idx).cuda()
    got = fx.topk_transform(t_idx, torch.from_numpy(table).cuda(), 1, row_base=torch.from_numpy(ks).cuda(),
                            row_table=torch.from_numpy(rt).cuda())
    assert np.array_equal(got.cpu().numpy(), want)
    fx.topk_transform(t_idx, torch.from_numpy(table).cuda(), 1, row_base=torch.from_numpy(ks).cuda(),
                      row_table=torch.from_numpy(rt).cuda(), out=t_idx)       # in place
    assert np.array_equal(t_idx.cpu().numpy(), want)


def test_transform_through_the_block_table_matches_oracle():
    """Seeded top-k positions of paged rows (R rows per request, -1 padding)
    through the paged form's block table of 64-token pages: GPU against oracle."""
    lengths = [5000, 300, 4200, 64, 2049]
    R, k = 4, 512
    d = workloads.make_paged(len(lengths), R, 1, 5000, seed=23, lengths=lengths)
    g = np.random.default_rng(29)
    idx = np.full((len(lengths) * R, k), -1, dtype=np.int32)
    for row in range(idx.shape[0]):
        L = lengths[row // R]
        n = min(k, L)
        idx[row, :n] = g.choice(L, size=n, replace=False)
    want = ip.topk_transform(idx, d["block_table"].numpy(), 64, rows_per_table_row=R)
    slots = fx.topk_transform(torch.from_numpy(idx).cuda(), d["block_table"].cuda(), 64, rows_per_table_row=R)
    assert np.array_equal(slots.cpu().numpy(), want)
    assert np.all((want >= 0) == (idx >= 0))


@pytest.mark.parametrize("lengths,R,k", [
    ([5000, 300, 4200, 64, 2049, 1, 129], 4, 2048),   # direct and short rows
    ([9000, 7000, 130, 6000], 8, 512),                # MTP-8, top-512
    ([3000] * 40, 1, 2048),                            # decode, many requests
    ([200 + (i % 7) * 37 for i in range(1200)], 1, 64),  # enough requests for whole-row units (no merge)
])
def test_paged_topk_slots_match_oracle(lengths, R, k):
    """The paged top-k written as physical KV slots (the transform applied
    where the indices are emitted, in the fused kernel or the merge): each
    slot maps back through the block table to a logical position that passes
    the oracle's top-k check, and equals the oracle's transform of it."""
    d = workloads.make_paged(len(lengths), R, 1, max(lengths), seed=31 + R, lengths=lengths)
    t = {x: d[x].cuda() for x in ("q", "k_pages", "s_pages", "w", "block_table", "seq_lens")}
    ws = fx.alloc_workspace(fx.paged_workspace_size(len(lengths), R, d["max_blocks"], k))
    slots, vals = fx.paged_mqa_logits_topk(**t, R=R, topk=k, return_values=True, workspace=ws, slots=True)
    assert fx.read_device_status(ws) == 0
    slots, vals = slots.cpu().numpy(), vals.cpu().numpy()
    bt = d["block_table"].numpy()
    rows = np.arange(len(lengths) * R)
    ref = paged_logits_rows(d["q"].numpy(), d["k_pages"].numpy(), d["s_pages"].numpy(), d["w"].numpy(), bt,
                            d["seq_lens"].numpy(), R, rows=rows)
    for row in rows:
        b = row // R
        L = int(lengths[b])
        page_to_block = {int(pg): blk for blk, pg in enumerate(bt[b, :(L + 63) // 64])}
        s = slots[row]
        pos = np.array([-1 if x < 0 else page_to_block[int(x) // 64] * 64 + int(x) % 64 for x in s],
                       dtype=np.int64)
        lo, hi = paged_range(L, R, row % R)
        check_topk_row(pos, ref[row], lo, hi, k, vals[row], f"row {row}")
        want = ip.topk_transform(pos[None, :].astype(np.int32), bt[b:b + 1], 64)
        assert np.array_equal(want[0], s), f"row {row}: slot differs from the oracle transform"
