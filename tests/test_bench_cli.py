"""Host-side checks of bench.py: argument rules and the pair count (no GPU)."""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_defaults_are_the_headline_run():
    a = bench.strict_args([])
    assert (a.gpus, a.impl, a.workload, a.path) == (1, "ours", bench.WORKLOAD, "fused")
    assert a.warmup >= 3


@pytest.mark.parametrize("argv", [
    ["--warmup", "2"],
    ["--steps", "0"],
    ["--gpus", "0"],
    ["--path", "chained", "--workload", "4"],      # the paged form has no chained path
    ["--path", "chained", "--impl", "reference"],
    ["--path", "act_quant"],                       # the key pool belongs to workload 4
    ["--path", "act_quant", "--workload", "4", "--impl", "reference"],
    ["--workload", "9"],
    ["--wark", "3"],                               # no prefix matching of options
])
def test_rejects(argv):
    with pytest.raises(SystemExit):
        bench.strict_args(argv)


def test_valid_pairs_clamps_ranges():
    ks = torch.tensor([0, -5, 10, 7], dtype=torch.int32)
    ke = torch.tensor([4, 3, 5, 100], dtype=torch.int32)
    # rows: [0,4) -> 4, [0,3) -> 3, empty -> 0, [7, n=20) -> 13
    assert bench.valid_pairs(ks, ke, 20) == 4 + 3 + 0 + 13


def test_chained_chunks_respect_the_logits_budget():
    n = 210000
    rows = max(1, bench.CHUNK_BYTES // (4 * n))
    assert rows * n * 4 <= bench.CHUNK_BYTES < (rows + 1) * n * 4
