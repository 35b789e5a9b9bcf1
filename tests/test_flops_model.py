"""The useful-work model against the pages' printed numbers and closed forms."""
import json
import os

import numpy as np

from long_context_index_b200 import flops

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "eq12_ratio.json")


def test_eq12_reproduces_printed_ratio():
    g = json.load(open(GOLDEN))
    f_gqa, f_msa = flops.eq12_flops(g["N"], g["H_q"], g["d_h"], g["H_kv"], g["d_idx"], g["k"], g["B_k"])
    assert round(f_gqa / f_msa, 1) == g["printed_ratio"]
    assert g["k"] * g["B_k"] == g["printed_budget_tokens"]


def test_visible_pairs_closed_form():
    assert flops.visible_pairs(1000, 1000, 0) == 1000 * 1001 // 2
    assert flops.visible_pairs(10, 100, 90) == sum(range(91, 101))
    assert flops.visible_pairs(7, 50, 0, causal=False) == 350


def test_selected_keys_counts_visible_keys_only():
    ids = np.array([[[0, 2, -1]], [[0, 1, 2]]], dtype=np.int32)   # rows at positions 40 and 41, B_k = 16
    # row 40: block 0 (16) + block 2 (keys 32..40 -> 9); row 41: 16 + 16 + 10
    assert flops.selected_keys(ids, 16, 64, 40) == 16 + 9 + 16 + 16 + 10


def test_index_and_main_flops_at_128k():
    n = 131072
    assert abs(flops.index_flops(n, n, 0, 4, 64) / 1e12 - 4.398) < 1e-3
    dense = flops.dense_main_flops(n, n, 0, 64, 128)
    assert abs(dense - 4 * 64 * 128 * n * (n + 1) / 2) < 1
