"""B200-native fp8 MQA indexer: logits + top-k over fp8 keys.

A thin Python binding over the C ABI of ``libfp8idx.so`` (``include/fp8idx.h``):
each function only checks and marshals torch CUDA tensors into pointers and
sizes and calls the entry point of the same name on the current CUDA stream.
Every arithmetic step runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and a missing or unloadable library raises.

  mqa_logits(q, k, s, w, ks, ke)                         -> logits [m, n] f32
  topk_rows(logits, ks, ke, topk)                        -> idx [m, topk] i32
  mqa_logits_topk(q, k, s, w, ks, ke, topk)              -> idx (and values)
  paged_mqa_logits_topk(q, k_pages, s_pages, w, block_table, seq_lens, R, topk)
  act_quant_store(x, slot_mapping, k_pages, s_pages)     bf16 keys -> fp8 key pool
  prepare_ragged(seq_len, q_len, req_idx, req_to_token, q_cap)  ragged ks/ke (+ index copy)
  topk_transform(idx, page_table, page_size, ...)        selected positions -> physical slots

q/k are fp8 e4m3fn bytes (torch.uint8 or torch.float8_e4m3fn), s/w float32,
ks/ke/block_table/seq_lens int32.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import workloads  # noqa: F401  (seeded synthetic inputs)

H = 32
D = 128
MAX_TOPK = 2048
PAGE_SIZE = 64

OK, EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA = 0, 1, 2, 3, 4
STATUS_WAIT_TIMEOUT, STATUS_BAD_PAGE, STATUS_SEQ_TOO_LONG = 1, 2, 4

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8idx.so")
_lock = threading.Lock()
_lib = None


class Fp8IdxError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"fp8idx error {code}: {msg}")
        self.code = code


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m fp8_mqa_logits_03_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
            L.fp8idx_mqa_logits.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i32, i32, vp, i64, vp]
            L.fp8idx_topk_rows.argtypes = [vp, i64, vp, vp, i64, i64, i32, vp, vp]
            L.fp8idx_mqa_logits_topk_workspace.argtypes = [i64, i64, i32, i32, i32]
            L.fp8idx_mqa_logits_topk_workspace.restype = sz
            L.fp8idx_mqa_logits_topk.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i32, i32, i32,
                                                 vp, vp, vp, sz, vp]
            L.fp8idx_paged_mqa_logits_topk_workspace.argtypes = [i64, i32, i32, i32, i32, i32]
            L.fp8idx_paged_mqa_logits_topk_workspace.restype = sz
            L.fp8idx_paged_mqa_logits_topk.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, i32, i64,
                                                       i32, i32, i32, i32, vp, vp, vp, sz, vp]
            L.fp8idx_paged_mqa_logits_topk_slots.argtypes = L.fp8idx_paged_mqa_logits_topk.argtypes
            L.fp8idx_read_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int), vp]
            L.fp8idx_read_device_stats.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32), i32, vp]
            L.fp8idx_read_device_stats.restype = ctypes.c_int
            L.fp8idx_last_error.restype = ctypes.c_char_p
            L.fp8idx_num_sms.restype = ctypes.c_int
            L.fp8idx_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
            L.fp8idx_debug_withhold_first_tile.argtypes = [ctypes.c_int]
            L.fp8idx_act_quant_store.argtypes = [vp, i64, i32, vp, i64, vp, vp, vp]
            L.fp8idx_prepare_ragged.argtypes = [vp, vp, vp, i32, vp, i64, i64, vp, vp, vp, i64, vp, i64,
                                                vp]
            L.fp8idx_topk_transform.argtypes = [vp, i64, i32, vp, vp, i32, vp, i64, i64, i32, vp, vp]
            for name in ("fp8idx_mqa_logits", "fp8idx_topk_rows", "fp8idx_mqa_logits_topk",
                         "fp8idx_paged_mqa_logits_topk", "fp8idx_paged_mqa_logits_topk_slots",
                         "fp8idx_read_device_status",
                         "fp8idx_act_quant_store", "fp8idx_prepare_ragged", "fp8idx_topk_transform"):
                getattr(L, name).restype = ctypes.c_int
            _lib = L
    return _lib


def _check(rc: int):
    if rc != OK:
        raise Fp8IdxError(rc, lib().fp8idx_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _bytes(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    if t.dtype != torch.uint8:
        raise TypeError(f"{name} must be fp8 e4m3fn bytes (uint8 or float8_e4m3fn), got {t.dtype}")
    return _dev(t, name)


def _dev(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def num_sms() -> int:
    return lib().fp8idx_num_sms()


def set_wait_limit_ns(ns: int) -> None:
    lib().fp8idx_set_wait_limit_ns(int(ns))


def debug_withhold_first_tile(on: bool) -> None:
    """Tests only: later fused / paged calls never load their first key tile,
    so a bounded wait runs out and the call reports WAIT_TIMEOUT."""
    lib().fp8idx_debug_withhold_first_tile(1 if on else 0)


# Names the library's fixed scratch array (the allocation-free entry point)
# where a workspace is expected by the diagnostics calls.
NOALLOC_WS = "noalloc"


def _ws_ptr(workspace):
    return ctypes.c_void_p(1) if isinstance(workspace, str) and workspace == NOALLOC_WS else _ptr(workspace)


def read_device_status(workspace=None, stream=None) -> int:
    """Status bits of the last call that used `workspace` (None: the last
    mqa_logits call; NOALLOC_WS: the last allocation-free call).  Synchronises."""
    v = ctypes.c_int(0)
    _check(lib().fp8idx_read_device_status(_ws_ptr(workspace), ctypes.byref(v), _stream(stream)))
    return v.value


def read_device_stats(workspace, stream=None) -> dict:
    """Counters the fused top-k left in a workspace's status block (tuning aid)."""
    buf = (ctypes.c_uint32 * 6)()
    _check(lib().fp8idx_read_device_stats(_ws_ptr(workspace), buf, 6, _stream(stream)))
    return dict(status=buf[0], compactions=buf[1], general_selects=buf[2], candidates=buf[3],
                max_boundary=buf[4], repairs=buf[5])


# ---------------------------------------------------------------------------- calls

def mqa_logits(q, k, s, w, ks, ke, logits=None, stream=None) -> torch.Tensor:
    """fp32 logits [m, n]: s[j] * sum_h w[i,h] * ReLU(q[i,h].k[j]) on [ks, ke), -inf elsewhere."""
    q = _bytes(q, "q")
    k = _bytes(k, "k")
    s = _dev(s, "s", torch.float32)
    w = _dev(w, "w", torch.float32)
    ks = _dev(ks, "ks", torch.int32)
    ke = _dev(ke, "ke", torch.int32)
    m, n = q.shape[0], k.shape[0]
    if logits is None:
        logits = torch.empty((m, n), dtype=torch.float32, device=q.device)
    if logits.dim() != 2 or logits.stride(1) != 1 or logits.dtype != torch.float32:
        raise ValueError("logits must be a [m, >=n] float32 tensor with unit column stride")
    _check(lib().fp8idx_mqa_logits(_ptr(q), _ptr(k), _ptr(s), _ptr(w), _ptr(ks), _ptr(ke), m, n,
                                   q.shape[1], q.shape[2], _ptr(logits), logits.stride(0),
                                   _stream(stream)))
    return logits


def topk_rows(logits, ks, ke, topk: int = MAX_TOPK, out=None, n=None, stream=None) -> torch.Tensor:
    """Top-k column indices of each logit row over [ks, ke) (ties: lower index), -1 padded."""
    logits = _dev(logits, "logits", torch.float32) if logits.stride(1) == 1 else None
    if logits is None:
        raise ValueError("logits must have unit column stride")
    ks = _dev(ks, "ks", torch.int32)
    ke = _dev(ke, "ke", torch.int32)
    m = logits.shape[0]
    n = logits.shape[1] if n is None else n
    if out is None:
        out = torch.empty((m, topk), dtype=torch.int32, device=logits.device)
    _check(lib().fp8idx_topk_rows(_ptr(logits), logits.stride(0), _ptr(ks), _ptr(ke), m, n, topk,
                                  _ptr(out), _stream(stream)))
    return out


def mqa_logits_topk_workspace_size(m: int, n: int, topk: int = MAX_TOPK, heads: int = H) -> int:
    return int(lib().fp8idx_mqa_logits_topk_workspace(m, n, heads, D, topk))


def paged_workspace_size(B: int, R: int, max_blocks: int, topk: int = MAX_TOPK, heads: int = H) -> int:
    return int(lib().fp8idx_paged_mqa_logits_topk_workspace(B, R, max_blocks, heads, D, topk))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A 256-byte aligned device buffer (torch's caching allocator aligns to 512)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8,
                       device=device if device is not None else "cuda")


def mqa_logits_topk(q, k, s, w, ks, ke, topk: int = MAX_TOPK, out=None, out_vals=None,
                    workspace=None, return_values: bool = False, stream=None):
    """Fused logits + top-k without materialising the m x n logits."""
    q = _bytes(q, "q")
    k = _bytes(k, "k")
    s = _dev(s, "s", torch.float32)
    w = _dev(w, "w", torch.float32)
    ks = _dev(ks, "ks", torch.int32)
    ke = _dev(ke, "ke", torch.int32)
    m, n = q.shape[0], k.shape[0]
    if out is None:
        out = torch.empty((m, topk), dtype=torch.int32, device=q.device)
    if return_values and out_vals is None:
        out_vals = torch.empty((m, topk), dtype=torch.float32, device=q.device)
    need = mqa_logits_topk_workspace_size(m, n, topk, q.shape[1])
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    _check(lib().fp8idx_mqa_logits_topk(_ptr(q), _ptr(k), _ptr(s), _ptr(w), _ptr(ks), _ptr(ke), m,
                                        n, q.shape[1], q.shape[2], topk, _ptr(out), _ptr(out_vals),
                                        _ptr(workspace), workspace.numel(), _stream(stream)))
    return (out, out_vals) if return_values else out


def paged_mqa_logits_topk(q, k_pages, s_pages, w, block_table, seq_lens, R: int,
                          topk: int = MAX_TOPK, out=None, out_vals=None, workspace=None,
                          return_values: bool = False, stream=None, slots: bool = False):
    """Paged decode/verify: R rows per request, keys through a 64-token block table.

    slots=True returns physical KV slots (block_table[b, j // 64] * 64 + j % 64)
    instead of logical positions j, mapped where the indices are written."""
    q = _bytes(q, "q")
    k_pages = _bytes(k_pages, "k_pages")
    s_pages = _dev(s_pages, "s_pages", torch.float32)
    w = _dev(w, "w", torch.float32)
    block_table = _dev(block_table, "block_table", torch.int32)
    seq_lens = _dev(seq_lens, "seq_lens", torch.int32)
    B, max_blocks = block_table.shape
    num_pages = k_pages.shape[0]
    page_size = k_pages.shape[1]
    rows = q.shape[0]
    if rows != B * R:
        raise ValueError(f"q has {rows} rows, expected B*R = {B * R}")
    if out is None:
        out = torch.empty((rows, topk), dtype=torch.int32, device=q.device)
    if return_values and out_vals is None:
        out_vals = torch.empty((rows, topk), dtype=torch.float32, device=q.device)
    need = paged_workspace_size(B, R, max_blocks, topk, q.shape[1])
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    fn = lib().fp8idx_paged_mqa_logits_topk_slots if slots else lib().fp8idx_paged_mqa_logits_topk
    _check(fn(_ptr(q), _ptr(k_pages), _ptr(s_pages), _ptr(w), _ptr(block_table), _ptr(seq_lens), B, R,
              max_blocks, num_pages, page_size, q.shape[1], q.shape[2], topk, _ptr(out), _ptr(out_vals),
              _ptr(workspace), workspace.numel(), _stream(stream)))
    return (out, out_vals) if return_values else out


def act_quant_store(x, slot_mapping, k_pages, s_pages, stream=None):
    """Quantise bf16 key rows into the fp8 key pool, in place.

    x [T, 128] bfloat16; slot_mapping [T] int64 (pool slot = page * 64 + row,
    a slot outside the pool is skipped); k_pages [P, 64, 128] uint8 (or
    float8_e4m3fn) and s_pages [P, 64] float32 receive the e4m3 codes and the
    per-token scale max(max |x|, 1e-4) / 448.
    """
    if not isinstance(x, torch.Tensor) or x.dtype != torch.bfloat16:
        raise TypeError("x must be a bfloat16 tensor")
    x = _dev(x, "x")
    slot_mapping = _dev(slot_mapping, "slot_mapping", torch.int64)
    k_pages = _bytes(k_pages, "k_pages")
    s_pages = _dev(s_pages, "s_pages", torch.float32)
    T = x.shape[0]
    num_slots = s_pages.numel()
    if x.dim() != 2 or slot_mapping.numel() != T or k_pages.numel() != num_slots * x.shape[1]:
        raise ValueError("x [T, D], slot_mapping [T], k_pages [slots, D] and s_pages [slots] disagree")
    _check(lib().fp8idx_act_quant_store(_ptr(x), T, x.shape[1], _ptr(slot_mapping), num_slots,
                                        _ptr(k_pages), _ptr(s_pages), _stream(stream)))
    return k_pages, s_pages


# ---------------------------------------------------------------------------- index preparation

def prepare_ragged(seq_len, q_len, req_idx, req_to_token, q_cap: int, ragged_cap: int = 0,
                   with_ragged: bool = True, ks=None, ke=None, row_table=None, ragged=None, stream=None):
    """Ragged key ranges of the batch's query rows (and its ragged token-slot
    buffer): fp8idx_prepare_ragged.  Returns (ks, ke, row_table, ragged or None)."""
    seq_len = _dev(seq_len, "seq_len", torch.int32)
    q_len = _dev(q_len, "q_len", torch.int32)
    req_idx = _dev(req_idx, "req_idx", torch.int32)
    req_to_token = _dev(req_to_token, "req_to_token", torch.int32)
    if req_to_token.dim() != 2:
        raise ValueError("req_to_token must be [rows, ld]")
    B = seq_len.numel()
    if q_len.numel() != B or req_idx.numel() != B:
        raise ValueError("seq_len, q_len and req_idx must have one entry per request")
    dev = seq_len.device
    ks = torch.empty(q_cap, dtype=torch.int32, device=dev) if ks is None else ks
    ke = torch.empty(q_cap, dtype=torch.int32, device=dev) if ke is None else ke
    row_table = torch.empty(q_cap, dtype=torch.int32, device=dev) if row_table is None else row_table
    if with_ragged and ragged is None:
        ragged = torch.empty(ragged_cap, dtype=torch.int32, device=dev)
    _check(lib().fp8idx_prepare_ragged(_ptr(seq_len), _ptr(q_len), _ptr(req_idx), B, _ptr(req_to_token),
                                       req_to_token.shape[0], req_to_token.stride(0), _ptr(ks), _ptr(ke),
                                       _ptr(row_table), q_cap, _ptr(ragged) if with_ragged else None,
                                       ragged.numel() if with_ragged else 0, _stream(stream)))
    return ks, ke, row_table, (ragged if with_ragged else None)


def topk_transform(idx, page_table, page_size: int = 1, row_base=None, row_table=None,
                   rows_per_table_row: int = 1, out=None, stream=None):
    """Selected positions -> physical slots through a page table
    (fp8idx_topk_transform); -1 stays -1.  out may be idx (in place)."""
    idx = _dev(idx, "idx", torch.int32)
    page_table = _dev(page_table, "page_table", torch.int32)
    if idx.dim() != 2 or page_table.dim() != 2:
        raise ValueError("idx must be [rows, topk] and page_table [rows, ld]")
    rows, k = idx.shape
    if row_base is not None:
        row_base = _dev(row_base, "row_base", torch.int32)
    if row_table is not None:
        row_table = _dev(row_table, "row_table", torch.int32)
    out = torch.empty_like(idx) if out is None else out
    _check(lib().fp8idx_topk_transform(_ptr(idx), rows, k, _ptr(row_base), _ptr(row_table),
                                       rows_per_table_row, _ptr(page_table), page_table.shape[0],
                                       page_table.stride(0), page_size, _ptr(out), _stream(stream)))
    return out
