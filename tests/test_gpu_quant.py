"""Key quantisation into the paged pool vs the oracle, byte for byte (needs a B200).

Codes and scales decide integers from fp32 arithmetic that both sides take
in fp32 (the scale, the quotient) before the same round-to-nearest-even
e4m3 rule, so every code byte and every scale must be equal.
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_mqa_logits_03_b200 as fx
from _parity import check_topk_row, paged_range

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp8_mqa_logits_03_b200 import build
    build.build()
    fx.lib()


def _bits(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("T,pages,seed", [(3000, 64, 31), (1, 1, 32), (777, 13, 33)])
def test_act_quant_store_matches_oracle_bytes(T, pages, seed):
    g = torch.Generator().manual_seed(seed)
    slots = pages * 64
    xs = torch.randn(T, 128, generator=g) * torch.logspace(-6, 3, T)[:, None]
    if T > 10:
        xs[3] = 0.0                       # the scale floor
        xs[4] = 1e-30                     # far below the floor
        xs[5, 9] = 3.0e38                 # near the bf16 maximum
        xs[6] = 448.0 * torch.sign(xs[6])  # quotients exactly +-448
    x = xs.to(torch.bfloat16)
    perm = torch.randperm(slots, generator=g)
    slot = perm[: min(T, slots)].to(torch.int64)
    if T > slots:
        slot = torch.cat([slot, torch.full((T - slots,), -1, dtype=torch.int64)])
    if T > 10:
        slot[1] = -1                      # not stored
        slot[2] = slots + 5               # outside the pool: not stored
    kp0 = np.full((slots, 128), 0xAB, np.uint8)
    sp0 = np.full((slots,), -7.0, np.float32)
    ref_k, ref_s = oracle.act_quant_store(_bits(x), slot.numpy(), slots, kp0.copy(), sp0.copy())

    kp = torch.from_numpy(kp0.copy()).view(pages, 64, 128).cuda()
    sp = torch.from_numpy(sp0.copy()).view(pages, 64).cuda()
    fx.act_quant_store(x.cuda(), slot.cuda(), kp, sp)
    torch.cuda.synchronize()
    got_k = kp.view(slots, 128).cpu().numpy()
    got_s = sp.view(slots).cpu().numpy()
    assert np.array_equal(got_s.view(np.uint32), ref_s.view(np.uint32))
    bad = np.argwhere(got_k != ref_k)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at slot/dim {bad[:4].tolist()}"


def test_act_quant_store_feeds_the_paged_indexer():
    """Keys quantised by the library and read back by the paged indexer give
    the oracle's result on the same pool."""
    g = torch.Generator().manual_seed(40)
    B, R, L = 2, 4, 300
    pages = 2 * ((L + 63) // 64)
    xk = (torch.randn(B * L, 128, generator=g) * 2).to(torch.bfloat16)
    bt = torch.randperm(pages, generator=g).to(torch.int32).view(B, -1)
    pos = torch.arange(L)
    slot = torch.cat([(bt[b, pos // 64].long() * 64 + pos % 64) for b in range(B)])
    kp = torch.zeros(pages, 64, 128, dtype=torch.uint8, device="cuda")
    sp = torch.zeros(pages, 64, dtype=torch.float32, device="cuda")
    fx.act_quant_store(xk.cuda(), slot.cuda(), kp, sp)
    q = torch.randn(B * R, 32, 128, generator=g).clamp(-2, 2).to(torch.float8_e4m3fn).view(torch.uint8)
    w = torch.rand(B * R, 32, generator=g)
    seq = torch.full((B,), L, dtype=torch.int32)
    idx = fx.paged_mqa_logits_topk(q.cuda(), kp, sp, w.cuda(), bt.cuda(), seq.cuda(), R=R, topk=64)
    torch.cuda.synchronize()
    ref_k, ref_s = oracle.act_quant_store(_bits(xk), slot.numpy(), pages * 64)
    assert np.array_equal(kp.view(-1, 128).cpu().numpy(), ref_k)
    lg = oracle.paged_logits_rows(q.numpy(), ref_k.reshape(pages, 64, 128), ref_s.reshape(pages, 64),
                                  w.numpy(), bt.numpy(), seq.numpy(), R)
    got = idx.cpu().numpy()
    for r in range(B * R):
        lo, hi = paged_range(L, R, r % R)
        check_topk_row(got[r], lg[r], lo, hi, 64, None, f"row {r}")
