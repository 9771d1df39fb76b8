"""Pins for the float64 CPU oracle (no GPU).

Each test checks the oracle against something other than itself: bytes and
values fixed by the e4m3fn format and printed on the pages, torch's own
e4m3fn cast (a library routine), exact integer arithmetic, hand-computed
logits, a torch float64 einsum, brute force over subsets and invariants of
the top-k.  A plausible slip anywhere in the oracle (a dropped ReLU, a
transposed operand, a wrong scale index, the wrong tie order, an off-by-one
in the ragged range) fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from fp8_mqa_logits_03_b200 import workloads

NEG_INF = -math.inf


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------
# codec
# ----------------------------------------------------------------------------

def test_decode_all_bytes_matches_torch():
    b = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(b)
    ref = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zeros survive
    assert math.copysign(1.0, ours[0x80]) == -1.0 and math.copysign(1.0, ours[0]) == 1.0


def test_roundtrip_all_finite_bytes():
    b = np.array([x for x in range(256) if x not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(oracle.e4m3_encode(oracle.e4m3_decode(b)), b)


def test_codec_golden(golden_dir):
    g = _load(golden_dir, "e4m3_codec.json")
    xs = np.array([c["x"] for c in g["encode"]], np.float64)
    want = np.array([c["byte"] for c in g["encode"]], np.uint8)
    got = oracle.e4m3_encode(xs)
    assert got.tolist() == want.tolist()
    assert int(oracle.e4m3_encode(np.array([np.nan]))[0]) == g["encode_nan"]["byte"]
    db = np.array([c["byte"] for c in g["decode"]], np.uint8)
    assert oracle.e4m3_decode(db).tolist() == [c["x"] for c in g["decode"]]
    assert np.all(np.isnan(oracle.e4m3_decode(np.array(g["decode_nan"], np.uint8))))


def test_encode_matches_torch_within_range():
    gen = torch.Generator().manual_seed(7)
    x = torch.cat([
        torch.randn(20000, generator=gen, dtype=torch.float64) * 3,
        torch.randn(5000, generator=gen, dtype=torch.float64) * 0.01,    # subnormals
        (torch.rand(5000, generator=gen, dtype=torch.float64) * 2 - 1) * 440,
    ])
    # torch rounds from float32; keep values exactly representable in float32
    x = x.to(torch.float32).to(torch.float64)
    ref = x.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x.numpy())
    assert np.array_equal(got, ref)
    # every midpoint between adjacent finite codes: ties go to the even code
    vals = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2
    codes = oracle.e4m3_encode(mids)
    lo = np.arange(0, 0x7E)
    assert np.array_equal(codes, np.where(lo % 2 == 0, lo, lo + 1).astype(np.uint8))


# ----------------------------------------------------------------------------
# logits
# ----------------------------------------------------------------------------

def test_dot_is_exact_against_int64():
    """H=1, w=1, s=1: the logit is max(dot, 0) and the dot is an exact integer
    multiple of 2^-18; compare bit for bit with an int64 evaluation."""
    gen = torch.Generator().manual_seed(3)
    m, n, Dm = 6, 50, 128
    # full byte range except NaN, so extreme magnitudes appear
    qb = torch.randint(0, 256, (m, 1, Dm), generator=gen, dtype=torch.int64)
    kb = torch.randint(0, 256, (n, Dm), generator=gen, dtype=torch.int64)
    qb[(qb & 0x7F) == 0x7F] = 0x7E
    kb[(kb & 0x7F) == 0x7F] = 0x7E
    qb = qb.to(torch.uint8).numpy()
    kb = kb.to(torch.uint8).numpy()
    ql = oracle.mqa_logits_rows(qb, kb, np.ones(n, np.float32), np.ones((m, 1), np.float32),
                                np.zeros(m, np.int32), np.full(m, n, np.int32))
    # integer evaluation: every finite e4m3 value times 2^9 is an integer
    qi = (oracle.e4m3_decode(qb) * 512).astype(np.int64)
    ki = (oracle.e4m3_decode(kb) * 512).astype(np.int64)
    assert np.array_equal(qi.astype(np.float64) / 512, oracle.e4m3_decode(qb))
    dots = qi[:, 0, :] @ ki.T  # int64, units of 2^-18
    want = np.maximum(dots, 0).astype(np.float64) * 2.0 ** -18
    assert np.array_equal(ql, want)


def test_tiny_golden(golden_dir):
    g = _load(golden_dir, "tiny_logits.json")
    for c in g["cases"]:
        q = np.array(c["q"], np.uint8)
        k = np.array(c["k"], np.uint8)
        s = np.array(c["s"], np.float32)
        w = np.array(c["w"], np.float32)
        ks = np.array(c["ks"], np.int32)
        ke = np.array(c["ke"], np.int32)
        lg = oracle.mqa_logits_rows(q, k, s, w, ks, ke)
        want = np.array([[NEG_INF if v == "-inf" else v for v in r] for r in c["logits"]])
        assert np.array_equal(lg, want), c["name"]
        idx, vals = oracle.topk_rows(lg, ks, ke, c["topk"])
        assert idx.tolist() == c["idx"], c["name"]


def _torch_logits(d):
    """Independent float64 evaluation with library routines (einsum, clamp)."""
    qf = torch.from_numpy(oracle.e4m3_decode(d["q"].numpy()))
    kf = torch.from_numpy(oracle.e4m3_decode(d["k"].numpy()))
    dots = torch.einsum("ihd,jd->ijh", qf, kf)
    lg = torch.einsum("ijh,ih->ij", dots.clamp_min(0), d["w"].double()) * d["s"].double()[None, :]
    n = kf.shape[0]
    j = torch.arange(n)[None, :]
    lo = d["ks"].long().clamp(min=0)[:, None]
    hi = d["ke"].long().clamp(max=n)[:, None]
    return torch.where((j >= lo) & (j < hi), lg, torch.tensor(NEG_INF, dtype=torch.float64)).numpy()


@pytest.mark.parametrize("seed", [0, 1])
def test_logits_match_torch_einsum(seed):
    m, n = 7, 53
    ks = np.array([0, 3, -5, 10, 52, 40, 0], np.int32)     # negative start is clamped
    ke = np.array([53, 20, 7, 10, 80, 30, 1], np.int32)    # empty, beyond-n and reversed rows
    d = workloads.make_prefill(m, n, seed, ks=ks, ke=ke, heads=4, dim=16)
    ours = oracle.mqa_logits_rows(d["q"].numpy(), d["k"].numpy(), d["s"].numpy(), d["w"].numpy(),
                                  ks, ke)
    ref = _torch_logits(d)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(ours), fin)
    assert np.allclose(ours[fin], ref[fin], rtol=1e-13, atol=1e-12)


def test_logits_full_shape_rows_against_einsum():
    """H=32, D=128 rows of the tiny workload against the library einsum."""
    d = workloads.make_workload(0)
    rows = np.array([0, 5, 15], np.int64)
    ours = oracle.mqa_logits_rows(d["q"].numpy(), d["k"].numpy(), d["s"].numpy(), d["w"].numpy(),
                                  d["ks"].numpy(), d["ke"].numpy(), rows=rows)
    sub = dict(q=d["q"][rows], k=d["k"], s=d["s"], w=d["w"][rows], ks=d["ks"][rows],
               ke=d["ke"][rows])
    ref = _torch_logits(sub)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(ours), fin)
    assert np.allclose(ours[fin], ref[fin], rtol=1e-13, atol=1e-10)


# ----------------------------------------------------------------------------
# top-k
# ----------------------------------------------------------------------------

def _brute_topk(vals, lo, hi, k):
    """The unique subset whose every member beats every non-member under
    (value desc, index asc), found by enumerating subsets."""
    cand = list(range(lo, hi))
    take = min(k, len(cand))

    def beats(a, b):
        return vals[a] > vals[b] or (vals[a] == vals[b] and a < b)

    found = []
    for sub in itertools.combinations(cand, take):
        rest = [j for j in cand if j not in sub]
        if all(beats(a, b) for a in sub for b in rest):
            found.append(set(sub))
    assert len(found) == 1
    return found[0]


def test_topk_brute_force_small():
    rng = np.random.default_rng(11)
    for trial in range(60):
        n = int(rng.integers(1, 11))
        # few distinct values so that ties are common
        vals = rng.integers(-3, 4, size=n).astype(np.float64) * 0.5
        lo = int(rng.integers(0, n))
        hi = int(rng.integers(lo, n + 1))
        k = int(rng.integers(1, 7))
        row = np.full(n, NEG_INF)
        row[lo:hi] = vals[lo:hi]
        idx, got_vals = oracle.topk_rows(row[None], np.array([lo], np.int32),
                                         np.array([hi], np.int32), k)
        idx = idx[0]
        want = _brute_topk(row, lo, hi, k)
        sel = [j for j in idx.tolist() if j >= 0]
        assert set(sel) == want
        assert len(sel) == min(k, hi - lo)
        assert all(j == -1 for j in idx.tolist()[len(sel):])
        # output order: value desc, index asc
        assert sel == sorted(sel, key=lambda j: (-row[j], j))


def test_topk_matches_stable_sort():
    rng = np.random.default_rng(5)
    m, n, k = 9, 300, 40
    lg = np.round(rng.normal(size=(m, n)) * 4) / 4  # many exact ties
    ks = rng.integers(-5, 100, size=m).astype(np.int32)
    ke = rng.integers(50, 320, size=m).astype(np.int32)
    idx, vals = oracle.topk_rows(lg, ks, ke, k)
    for i in range(m):
        lo, hi = max(int(ks[i]), 0), min(int(ke[i]), n)
        hi = max(hi, lo)
        seg = torch.from_numpy(lg[i, lo:hi])
        order = torch.sort(-seg, stable=True).indices.numpy() + lo
        want = order[:k].tolist()
        want += [-1] * (k - len(want))
        assert idx[i].tolist() == want


def test_topk_invariants_on_tiny_workload():
    d = workloads.make_workload(0)
    k = workloads.TOPK
    idx, vals, lg = oracle.mqa_logits_topk_rows(d["q"].numpy(), d["k"].numpy(), d["s"].numpy(),
                                                d["w"].numpy(), d["ks"].numpy(), d["ke"].numpy(),
                                                k)
    n = d["n"]
    for i in range(d["m"]):
        lo, hi = int(d["ks"][i]), int(d["ke"][i])
        sel = idx[i][idx[i] >= 0]
        assert len(sel) == min(k, hi - lo)
        assert len(set(sel.tolist())) == len(sel)
        assert np.all((sel >= lo) & (sel < hi))
        if hi - lo >= k:
            assert np.all(idx[i] >= 0)           # -1 only when the range is short
        mask = np.zeros(n, bool)
        mask[sel] = True
        inside = np.zeros(n, bool)
        inside[lo:hi] = True
        unsel = lg[i][inside & ~mask]
        if unsel.size:
            assert lg[i][sel].min() >= unsel.max()
        assert np.array_equal(vals[i][: len(sel)], lg[i][sel])


# ----------------------------------------------------------------------------
# paged form
# ----------------------------------------------------------------------------

def test_paged_equals_prefill_on_gathered_keys():
    """Resolving the block table by hand and running the prefill form gives
    the paged form's logits and top-k exactly."""
    B, R, ps = 3, 4, 64
    d = workloads.make_paged(B, R, 70, 400, seed=9, page_size=ps, heads=32, dim=128)
    bt = d["block_table"].numpy()
    L = d["seq_lens"].numpy()
    kp = d["k_pages"].numpy()
    sp = d["s_pages"].numpy()
    lmax = int(L.max())
    k = 100
    pl = oracle.paged_logits_rows(d["q"].numpy(), kp, sp, d["w"].numpy(), bt, L, R)
    pidx, _ = oracle.paged_topk_rows(pl, L, R, k, np.arange(B * R))
    for b in range(B):
        keys = np.concatenate([kp[bt[b, p]] for p in range((L[b] + ps - 1) // ps)])[: L[b]]
        sc = np.concatenate([sp[bt[b, p]] for p in range((L[b] + ps - 1) // ps)])[: L[b]]
        ke = np.array([L[b] - R + t + 1 for t in range(R)], np.int32)
        ks = np.zeros(R, np.int32)
        rows = slice(b * R, (b + 1) * R)
        lg = oracle.mqa_logits_rows(d["q"].numpy()[rows], keys, sc, d["w"].numpy()[rows], ks, ke)
        assert np.array_equal(lg, pl[rows, : L[b]])
        assert np.all(np.isneginf(pl[rows, L[b]:lmax]))
        idx, _ = oracle.topk_rows(lg, ks, ke, k)
        assert np.array_equal(idx, pidx[rows])


def test_workload_shapes():
    for i, shape in workloads.WORKLOADS.items():
        if isinstance(shape, workloads.PrefillShape):
            if shape.m * shape.n > 10**8:
                continue
            d = workloads.make_workload(i)
            assert d["q"].shape == (shape.m, 32, 128) and d["k"].shape == (shape.n, 128)
            assert int(d["ke"].max()) <= shape.n and int(d["ks"].min()) == 0
    d = workloads.make_paged(5, 4, 4096, 8192, seed=1)
    bt = d["block_table"]
    used = bt[bt >= 0]
    assert used.numel() == d["P"] and torch.unique(used).numel() == d["P"]
    assert int(d["seq_lens"].min()) >= 4096 and int(d["seq_lens"].max()) <= 8192


# ---------------------------------------------------------------------------- key quantisation

def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def test_act_quant_unit_scale_row_is_the_codec():
    # amax exactly 448 gives the scale 1, so the codes are the codec itself
    g = torch.Generator().manual_seed(5)
    row = (torch.rand(128, generator=g) * 800 - 400)
    row[17] = -448.0
    x = _bf16_bits(row[None])
    kp, sp = oracle.act_quant_store(x, np.array([0]), 1)
    assert sp[0] == np.float32(1.0)
    xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).float().numpy()[0]
    assert np.array_equal(kp[0], oracle.e4m3_encode(xf.astype(np.float64)))
    assert kp[0, 17] == 0xFE  # -448


def test_act_quant_zero_row_uses_the_floor():
    kp, sp = oracle.act_quant_store(np.zeros((1, 128), np.uint16), np.array([0]), 1)
    assert sp[0] == np.float32(np.float32(1e-4) / np.float32(448.0))
    assert not kp.any()


def test_act_quant_matches_torch_fp32_and_its_e4m3_cast():
    # the same rule written with torch ops: fp32 amax, scale and quotient,
    # then torch's own float -> float8_e4m3fn cast (round to nearest even)
    g = torch.Generator().manual_seed(6)
    xs = torch.randn(300, 128, generator=g) * torch.logspace(-6, 3, 300)[:, None]
    xs[5] = 0.0
    xs[6, :] = 1e-30
    x = _bf16_bits(xs)
    xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).float()
    amax = xf.abs().amax(dim=1).clamp(min=1e-4)
    sc = amax / 448.0
    codes = (xf / sc[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    kp, sp = oracle.act_quant_store(x, np.arange(300), 300)
    assert np.array_equal(sp, sc.numpy())
    assert np.array_equal(kp, codes)


def test_act_quant_slots_and_error_bound():
    g = torch.Generator().manual_seed(7)
    xs = torch.randn(40, 128, generator=g) * 3
    x = _bf16_bits(xs)
    slot = np.array([(7 * t) % 64 for t in range(40)], np.int64)
    slot[3] = -1            # not stored
    slot[9] = 64            # outside the pool: not stored
    kp0 = np.full((64, 128), 0xAB, np.uint8)
    sp0 = np.full((64,), -7.0, np.float32)
    kp, sp = oracle.act_quant_store(x, slot, 64, kp0.copy(), sp0.copy())
    stored = {int(s) for s in slot if 0 <= s < 64}
    for s in range(64):
        if s not in stored:
            assert np.all(kp[s] == 0xAB) and sp[s] == np.float32(-7.0)
    xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).double().numpy()
    for t in range(40):
        s = int(slot[t])
        if not 0 <= s < 64:
            continue
        deq = oracle.e4m3_decode(kp[s]) * float(sp[s])
        # e4m3 keeps 3 mantissa bits: half an ulp is 2^-4 relative, or 2^-10 * scale below 2^-6
        assert np.all(np.abs(deq - xf[t]) <= 2.0 ** -4 * np.abs(xf[t]) + 2.0 ** -10 * float(sp[s]) + 1e-30)
