"""Float64 CPU oracle for the fp8 MQA indexer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library
and its binding in ``fp8_mqa_logits_03_b200``) never imports, links or runs
it, and the two share no code.

The arithmetic lives in ``fp8idx_oracle.c`` (plain C, float64).  This module
compiles it with gcc on first use and exposes it through ctypes with numpy
arrays.  See the C file's header for what is computed and which passage of
the pages each step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8idx_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc, no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-shared", "-fPIC",
               "-pthread", _SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            vp = ctypes.c_void_p
            lib.oracle_e4m3_decode.restype = ctypes.c_double
            lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
            lib.oracle_e4m3_decode_array.argtypes = [vp, ctypes.c_int64, vp]
            lib.oracle_e4m3_encode_array.argtypes = [vp, ctypes.c_int64, vp]
            lib.oracle_mqa_logits_rows.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int64,
                                                   ctypes.c_int64, ctypes.c_int, ctypes.c_int, vp,
                                                   ctypes.c_int64, vp, ctypes.c_int]
            lib.oracle_topk_rows.argtypes = [vp, ctypes.c_int64, vp, vp, vp, ctypes.c_int64,
                                             ctypes.c_int, vp, vp]
            lib.oracle_paged_logits_rows.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int,
                                                     ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                     ctypes.c_int, ctypes.c_int, vp, ctypes.c_int64,
                                                     ctypes.c_int64, vp, ctypes.c_int]
            lib.oracle_paged_topk_rows.argtypes = [vp, ctypes.c_int64, vp, ctypes.c_int, vp,
                                                   ctypes.c_int64, ctypes.c_int, vp, vp]
            lib.oracle_act_quant_store.argtypes = [vp, ctypes.c_int64, ctypes.c_int, vp,
                                                   ctypes.c_int64, vp, vp]
            _lib = lib
    return _lib


def host_threads() -> int:
    """Number of host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


# ----------------------------------------------------------------------------
# codec
# ----------------------------------------------------------------------------

def e4m3_decode(b) -> np.ndarray:
    """fp8 e4m3fn bytes -> float64 (exact)."""
    lib = _load()
    a = _c(np.asarray(b), np.uint8)
    out = np.empty(a.shape, np.float64)
    lib.oracle_e4m3_decode_array(_p(a), a.size, _p(out))
    return out


def e4m3_encode(x) -> np.ndarray:
    """float64 -> fp8 e4m3fn bytes: round-to-nearest-even, saturating at +-448."""
    lib = _load()
    a = _c(np.asarray(x), np.float64)
    out = np.empty(a.shape, np.uint8)
    lib.oracle_e4m3_encode_array(_p(a), a.size, _p(out))
    return out


# ----------------------------------------------------------------------------
# prefill form
# ----------------------------------------------------------------------------

def mqa_logits_rows(q, k, s, w, ks, ke, rows=None, threads: int | None = None) -> np.ndarray:
    """float64 logits for the listed query rows: shape [len(rows), n], -inf outside [ks, ke).

    q: [m, H, D] uint8 (e4m3 bytes); k: [n, D] uint8; s: [n] f32; w: [m, H] f32;
    ks, ke: [m] int32.
    """
    lib = _load()
    q = _c(q, np.uint8)
    k = _c(k, np.uint8)
    s = _c(s, np.float32)
    w = _c(w, np.float32)
    ks = _c(ks, np.int32)
    ke = _c(ke, np.int32)
    m, H, D = q.shape
    n = k.shape[0]
    rows = np.arange(m, dtype=np.int64) if rows is None else _c(rows, np.int64)
    out = np.empty((rows.size, n), np.float64)
    lib.oracle_mqa_logits_rows(_p(q), _p(k), _p(s), _p(w), _p(ks), _p(ke), m, n, H, D, _p(rows),
                               rows.size, _p(out), threads or host_threads())
    return out


def topk_rows(logits, ks, ke, k: int, rows=None):
    """Top-k of logit rows (row r uses ks/ke of query row rows[r]).

    Returns (idx [nrows, k] int32 padded with -1, vals [nrows, k] float64 padded with -inf).
    """
    lib = _load()
    logits = _c(logits, np.float64)
    ks = _c(ks, np.int32)
    ke = _c(ke, np.int32)
    nrows, n = logits.shape
    rows = np.arange(nrows, dtype=np.int64) if rows is None else _c(rows, np.int64)
    idx = np.empty((nrows, k), np.int32)
    vals = np.empty((nrows, k), np.float64)
    lib.oracle_topk_rows(_p(logits), n, _p(ks), _p(ke), _p(rows), nrows, k, _p(idx), _p(vals))
    return idx, vals


def mqa_logits_topk_rows(q, k, s, w, ks, ke, topk: int, rows=None, threads: int | None = None):
    """Logits then top-k for the listed rows: (idx, vals, logits)."""
    m = np.asarray(q).shape[0]
    rows = np.arange(m, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    lg = mqa_logits_rows(q, k, s, w, ks, ke, rows, threads)
    idx, vals = topk_rows(lg, ks, ke, topk, rows)
    return idx, vals, lg


# ----------------------------------------------------------------------------
# paged form
# ----------------------------------------------------------------------------

def paged_logits_rows(q, k_pages, s_pages, w, block_table, seq_lens, R: int, rows=None,
                      lmax: int | None = None, threads: int | None = None) -> np.ndarray:
    """float64 logits of the paged form for global rows (row = b*R + t): [len(rows), lmax]."""
    lib = _load()
    q = _c(q, np.uint8)
    k_pages = _c(k_pages, np.uint8)
    s_pages = _c(s_pages, np.float32)
    w = _c(w, np.float32)
    block_table = _c(block_table, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    BR, H, D = q.shape
    B, max_blocks = block_table.shape
    page_size = k_pages.shape[1]
    if lmax is None:
        lmax = int(seq_lens.max()) if seq_lens.size else 0
    rows = np.arange(BR, dtype=np.int64) if rows is None else _c(rows, np.int64)
    out = np.empty((rows.size, lmax), np.float64)
    lib.oracle_paged_logits_rows(_p(q), _p(k_pages), _p(s_pages), _p(w), _p(block_table),
                                 _p(seq_lens), B, R, max_blocks, page_size, H, D, _p(rows),
                                 rows.size, lmax, _p(out), threads or host_threads())
    return out


def paged_topk_rows(logits, seq_lens, R: int, k: int, rows):
    lib = _load()
    logits = _c(logits, np.float64)
    seq_lens = _c(seq_lens, np.int32)
    rows = _c(rows, np.int64)
    nrows, lmax = logits.shape
    idx = np.empty((nrows, k), np.int32)
    vals = np.empty((nrows, k), np.float64)
    lib.oracle_paged_topk_rows(_p(logits), lmax, _p(seq_lens), R, _p(rows), nrows, k, _p(idx),
                               _p(vals))
    return idx, vals


def paged_logits_topk_rows(q, k_pages, s_pages, w, block_table, seq_lens, R: int, topk: int,
                           rows=None, threads: int | None = None):
    BR = np.asarray(q).shape[0]
    rows = np.arange(BR, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    lg = paged_logits_rows(q, k_pages, s_pages, w, block_table, seq_lens, R, rows, None, threads)
    idx, vals = paged_topk_rows(lg, seq_lens, R, topk, rows)
    return idx, vals, lg


# ----------------------------------------------------------------------------
# key quantisation into the paged pool
# ----------------------------------------------------------------------------

def act_quant_store(x_bf16, slot, num_slots: int, k_pool=None, s_pool=None):
    """Quantise bf16 key rows to e4m3 with one fp32 scale per token and store
    them in a pool of `num_slots` 128-byte slots (64 per page).

    x_bf16: [T, D] uint16 (bf16 bit patterns); slot: [T] int64, a slot outside
    [0, num_slots) is skipped.  k_pool [num_slots, D] uint8 and s_pool
    [num_slots] f32 are updated in place (created zero-filled when None) and
    returned.  s_t = max(max_d |x_t|, 1e-4) / 448 and codes = e4m3(x / s_t),
    both in fp32.
    """
    lib = _load()
    x = _c(x_bf16, np.uint16)
    slot = _c(slot, np.int64)
    T, D = x.shape
    if k_pool is None:
        k_pool = np.zeros((num_slots, D), np.uint8)
    if s_pool is None:
        s_pool = np.zeros((num_slots,), np.float32)
    assert k_pool.flags.c_contiguous and k_pool.dtype == np.uint8 and k_pool.shape == (num_slots, D)
    assert s_pool.flags.c_contiguous and s_pool.dtype == np.float32 and s_pool.shape == (num_slots,)
    lib.oracle_act_quant_store(_p(x), T, D, _p(slot), num_slots, _p(k_pool), _p(s_pool))
    return k_pool, s_pool
