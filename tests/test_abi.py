"""The C ABI without a GPU: the library loads, exports every entry point that
include/fp8idx.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import fp8_mqa_logits_03_b200 as fx
from fp8_mqa_logits_03_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return fx.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "fp8idx.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8idx_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    syms = declared_symbols()
    assert len(syms) >= 10
    for name in syms:
        assert hasattr(L, name), name


FAKE = ctypes.c_void_p(4096)        # never dereferenced: validation fails first
MIS = ctypes.c_void_p(4096 + 4)     # 4-byte aligned, not 16-byte aligned


def _fused(L, q=FAKE, k=FAKE, m=8, n=64, H=32, D=128, topk=16, out=FAKE, ws=FAKE, ws_bytes=1 << 20):
    return L.fp8idx_mqa_logits_topk(q, k, FAKE, FAKE, FAKE, FAKE, m, n, H, D, topk, out, None, ws,
                                    ws_bytes, None)


def test_rejects_before_launch(L):
    assert _fused(L, H=16) == fx.EUNSUPPORTED
    assert _fused(L, D=64) == fx.EUNSUPPORTED
    assert _fused(L, topk=0) == fx.EINVAL
    assert _fused(L, topk=2049) == fx.EINVAL
    assert _fused(L, m=-1) == fx.EINVAL
    assert _fused(L, n=-5) == fx.EINVAL
    assert _fused(L, q=None) == fx.EINVAL
    assert _fused(L, q=MIS) == fx.EINVAL
    assert _fused(L, k=MIS) == fx.EINVAL
    assert b"16-byte" in L.fp8idx_last_error()
    assert _fused(L, m=0) == fx.OK          # no-op
    assert L.fp8idx_last_error() == b""


def test_logits_and_topk_rows_reject(L):
    assert L.fp8idx_mqa_logits(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 10, 32, 128, FAKE, 5, None) == fx.EINVAL
    assert L.fp8idx_mqa_logits(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 10, 8, 128, FAKE, 10, None) == fx.EUNSUPPORTED
    assert L.fp8idx_mqa_logits(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 10, 32, 128, FAKE, 10, None) == fx.OK
    assert L.fp8idx_topk_rows(FAKE, 5, FAKE, FAKE, 3, 10, 16, FAKE, None) == fx.EINVAL   # ld < n
    assert L.fp8idx_topk_rows(FAKE, 10, FAKE, FAKE, 3, 10, 0, FAKE, None) == fx.EINVAL
    assert L.fp8idx_topk_rows(FAKE, 10, FAKE, FAKE, 0, 10, 16, FAKE, None) == fx.OK


@pytest.mark.parametrize("entry", ["fp8idx_paged_mqa_logits_topk", "fp8idx_paged_mqa_logits_topk_slots"])
def test_paged_rejects(L, entry):
    def call(R=4, page_size=64, H=32, B=2, max_blocks=4, num_pages=8, topk=64, q=FAKE, s_pages=FAKE):
        return getattr(L, entry)(q, FAKE, s_pages, FAKE, FAKE, FAKE, B, R, max_blocks,
                                 num_pages, page_size, H, 128, topk, FAKE, None, FAKE, 1 << 20, None)
    assert call(R=0) == fx.EUNSUPPORTED
    assert call(R=9) == fx.EUNSUPPORTED
    assert call(page_size=32) == fx.EUNSUPPORTED
    assert call(H=48) == fx.EUNSUPPORTED
    assert call(H=64, R=5) == fx.EUNSUPPORTED    # 64 heads: at most 4 rows per request
    assert call(max_blocks=0) == fx.EINVAL
    assert call(q=MIS) == fx.EINVAL
    assert call(s_pages=MIS) == fx.EINVAL        # page scales are bulk-copied: 16-byte aligned
    assert b"16-byte" in L.fp8idx_last_error()
    assert call(B=0) == fx.OK


def test_workspace_queries_reject_bad_shapes(L):
    assert L.fp8idx_mqa_logits_topk_workspace(8, 100, 32, 128, 0) == 0
    assert L.fp8idx_paged_mqa_logits_topk_workspace(4, 9, 16, 32, 128, 2048) == 0
    assert L.fp8idx_paged_mqa_logits_topk_workspace(4, 5, 16, 64, 128, 2048) == 0
    assert L.fp8idx_mqa_logits_topk_workspace(8, 100, 48, 128, 16) == 0


def test_act_quant_store_rejects(L):
    def call(x=FAKE, T=4, D=128, slot=FAKE, slots=64, kp=FAKE, sp=FAKE):
        return L.fp8idx_act_quant_store(x, T, D, slot, slots, kp, sp, None)
    assert call(D=64) == fx.EUNSUPPORTED
    assert call(T=-1) == fx.EINVAL
    assert call(slots=-1) == fx.EINVAL
    assert call(x=None) == fx.EINVAL
    assert call(slot=MIS) == fx.EINVAL          # int64 slots: 8-byte aligned
    assert call(x=MIS) == fx.EINVAL             # 4 bf16 per lane: 8-byte aligned
    assert call(kp=ctypes.c_void_p(4096 + 2)) == fx.EINVAL
    assert call(T=0) == fx.OK
