"""Pins of the oracle's index projections against facts fixed by
construction: a one-hot hidden state selects one column of every stacked
weight block (which pins the row split into the h_kv group query projections
and the shared key projection, and the transpose), and sums of one-hot rows
give sums of columns."""
import numpy as np

import oracle
from synth import f32_to_bf16_bits, make_index_projection


def test_one_hot_rows_select_weight_columns():
    h_kv, d_idx, d_model = 3, 4, 10
    w = np.arange((h_kv + 1) * d_idx * d_model, dtype=np.float32).reshape((h_kv + 1) * d_idx, d_model) % 97 - 48
    x = np.eye(d_model, dtype=np.float32)[[2, 7, 0]]
    q, k = oracle.index_project(f32_to_bf16_bits(x), f32_to_bf16_bits(w), h_kv, d_idx)
    for i, j in enumerate([2, 7, 0]):
        for r in range(h_kv):
            assert np.array_equal(q[i, r], w[r * d_idx:(r + 1) * d_idx, j])
        assert np.array_equal(k[i, 0], w[h_kv * d_idx:, j])


def test_row_sums_give_column_sums_and_integer_inputs_stay_exact():
    t = make_index_projection(3, 16, 64, 2, 8, integer=True)
    x = (t["x"].astype(np.uint32) << 16).view(np.float32)
    w = (t["w_idx"].astype(np.uint32) << 16).view(np.float32)
    assert np.all(np.count_nonzero(x, axis=1) == 8)
    q, k = oracle.index_project(t["x"], t["w_idx"], 2, 8)
    for i in range(16):
        cols = np.nonzero(x[i])[0]
        want = sum(x[i, c] * w[:, c].astype(np.float64) for c in cols)
        assert np.array_equal(np.concatenate([q[i].ravel(), k[i].ravel()]), want)
    assert np.all(np.abs(q) <= 24) and np.all(q == np.round(q))
