"""Index preparation and the top-k transform on the GPU against the oracle,
bit for bit (needs a B200).  Integer work: every output must be identical."""
import numpy as np
import pytest
import torch

from oracle import index_prep as ip
import fp8_mqa_logits_03_b200 as fx
from fp8_mqa_logits_03_b200 import workloads

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


def test_transform_of_the_paged_topk_matches_oracle():
    """The paged indexer's logical positions through its block table (64-token
    pages): the kernel's own output, transformed on the GPU and by the oracle."""
    lengths = [5000, 300, 4200, 64, 2049]
    R, k = 4, 512
    d = workloads.make_paged(len(lengths), R, 1, 5000, seed=23, lengths=lengths)
    t = {x: d[x].cuda() for x in ("q", "k_pages", "s_pages", "w", "block_table", "seq_lens")}
    idx = fx.paged_mqa_logits_topk(**t, R=R, topk=k)
    slots = fx.topk_transform(idx, t["block_table"], 64, rows_per_table_row=R)
    want = ip.topk_transform(idx.cpu().numpy(), d["block_table"].numpy(), 64, rows_per_table_row=R)
    assert np.array_equal(slots.cpu().numpy(), want)
    assert np.all((slots.cpu().numpy() >= 0) == (idx.cpu().numpy() >= 0))
