"""GPU parity of the index projections (msa_index_project) against the fp64
oracle, and of the chain projection -> index branch.

Tolerance, from the arithmetic: the tensor cores multiply bf16 exactly and
accumulate in fp32 (relative error per addition <= 2^-24, so |err| <=
d_model * 2^-24 * sum_t |x_t w_t| at worst), and the result is rounded to bf16
(half an ulp: 2^-9 |y|).  The test allows 2^-8 |y| + 2^-13 sum_t |x_t w_t|
(for d_model <= 8192 the accumulation bound is <= 2^-11 of the sum; observed
errors are far below it)."""
import numpy as np
import pytest
import torch

import long_context_index_b200 as msa
import oracle
from synth import make_index_projection
from tests.gpu_util import dev, host_f64, params_pair

pytestmark = pytest.mark.gpu


def widen(bits):
    return (np.ascontiguousarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def run_case(n, d_model, h_kv, d_idx, seed, integer=False):
    t = make_index_projection(seed, n, d_model, h_kv, d_idx, integer=integer)
    p, _ = params_pair(h_kv * 4, h_kv, 64, d_idx, 128, 8)
    q, k = msa.index_project(p, dev(t["x"]), dev(t["w_idx"]))
    torch.cuda.synchronize()
    q_ref, k_ref = oracle.index_project(t["x"], t["w_idx"], h_kv, d_idx)
    got = np.concatenate([host_f64(q).reshape(n, -1), host_f64(k).reshape(n, -1)], axis=1)
    ref = np.concatenate([q_ref.reshape(n, -1), k_ref.reshape(n, -1)], axis=1)
    if integer:
        assert np.array_equal(got, ref)
    else:
        mag = np.abs(widen(t["x"])) @ np.abs(widen(t["w_idx"])).T
        bad = np.abs(got - ref) > 2.0 ** -8 * np.abs(ref) + 2.0 ** -13 * mag
        assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:4].tolist())
    return t, q, k


@pytest.mark.parametrize("n,d_model,h_kv,d_idx", [
    (1000, 8192, 4, 64),      # model shape (hidden width h_q * d = 8192), ragged last row tile
    (129, 4096, 4, 64),
    (1, 1024, 4, 64),         # one row
    (300, 520, 2, 32),        # d_model not a multiple of the 64-column K slice; 96 output columns
    (257, 2048, 8, 128),      # 1152 output columns: three passes (512, 512, 128)
])
def test_projection_matches_oracle(n, d_model, h_kv, d_idx):
    run_case(n, d_model, h_kv, d_idx, seed=n + d_model)


def test_projection_then_index_branch_bit_exact():
    # Integer-valued x and weights make the projection exact, so the index
    # ids downstream must match the oracle's chain bit for bit.
    n, d_model, h_kv, d_idx = 3000, 8192, 4, 64
    t, q, k = run_case(n, d_model, h_kv, d_idx, seed=11, integer=True)
    p, po = params_pair(64, h_kv, 128, d_idx, 128, 16)
    ids = msa.index_topk(p, q, k)
    torch.cuda.synchronize()
    q_ref, k_ref = oracle.index_project(t["x"], t["w_idx"], h_kv, d_idx)
    from synth import f32_to_bf16_bits
    rows = np.r_[0:40, 1000:1040, n - 40:n]
    ids_ref = oracle.index_topk(po, f32_to_bf16_bits(q_ref.astype(np.float32)),
                                f32_to_bf16_bits(k_ref.astype(np.float32)), rows=rows)
    assert np.array_equal(ids.cpu().numpy()[rows], ids_ref)
