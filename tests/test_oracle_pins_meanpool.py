"""Pins of the oracle's mean-pool variant of the index branch (the MoBA-style
mean pooling that the m.163.com post compares with the block max-pool): the
pooled score of a block is the mean of the token scores of its visible keys.

Each expected value is fixed by construction, by an invariant, or by numpy
(a library matmul and mean) on tiny inputs with exhaustive subset search --
never by the oracle itself.
"""
import math

import numpy as np
import pytest

import oracle
from synth import bf16_bits_to_f32, f32_to_bf16_bits
from tests.test_oracle_pins import brute_force_select

MEAN = oracle.POOL_MEAN


def bf(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def P(**kw):
    base = dict(h_q=4, h_kv=2, d=8, d_idx=4, block_k=4, topk=3, causal=1, force_local=1, pool=MEAN)
    base.update(kw)
    return oracle.params(**base)


def line_inputs(vals, d_idx=4):
    """Q_idx[i, 0] = e_0 and K_idx[j, 0, 0] = vals[j]: token score j is vals[j] / sqrt(d_idx)."""
    n = len(vals)
    q = np.zeros((n, 1, d_idx), np.float32)
    q[:, 0, 0] = 1
    k = np.zeros((n, 1, d_idx), np.float32)
    k[:, 0, 0] = vals
    return bf(q), bf(k)


def test_block_mean_closed_form_causal():
    vals = [1, 2, 3, 6, -4, 0, 2, 2, 9, -1, 3, 1]
    B = 4
    q, k = line_inputs(vals)
    M = oracle.block_scores(P(h_q=1, h_kv=1, block_k=B), q, k)
    s = 1.0 / math.sqrt(4)
    for i in range(len(vals)):
        for b in range(len(vals) // B):
            vis = [vals[j] for j in range(b * B, (b + 1) * B) if j <= i]
            want = float(np.float32(sum(vis) / len(vis))) * s if vis else -np.inf
            assert M[i, 0, b] == want, (i, b, M[i, 0, b], want)


def test_mean_and_max_pool_pick_different_blocks():
    # Block 0 has one strong key among weak ones (high max, low mean); block 1
    # is uniformly medium (higher mean, lower max).  Mean pooling picks block 1,
    # max pooling block 0.
    vals = [-3, -3, 12, -3, 3, 3, 3, 3, 0, 0, 0, 0]
    q, k = line_inputs(vals)
    mean_ids = oracle.index_topk(P(h_q=1, h_kv=1, topk=2), q, k)
    max_ids = oracle.index_topk(P(h_q=1, h_kv=1, topk=2, pool=oracle.POOL_MAX), q, k)
    assert list(mean_ids[11, 0]) == [1, 2]
    assert list(max_ids[11, 0]) == [0, 2]


def test_partial_local_block_averages_visible_keys_only():
    # Query 9 sees keys 8 and 9 of block 2 (mean 0); keys 10 and 11 (not
    # visible) would raise the block's mean above block 0's if they counted.
    vals = [1, 1, 1, 1, -5, -5, -5, -5, 0, 0, 40, 40]
    q, k = line_inputs(vals)
    ids = oracle.index_topk(P(h_q=1, h_kv=1, topk=1, force_local=0), q, k)
    assert list(ids[9, 0]) == [0]
    M = oracle.block_scores(P(h_q=1, h_kv=1, force_local=0), q, k)
    assert M[9, 0, 2] == 0.0 and M[11, 0, 2] == 20.0 / 2


def test_mean_never_exceeds_max_and_equals_it_on_constant_blocks():
    rng = np.random.default_rng(3)
    q = bf(rng.integers(-3, 4, (64, 2, 8)))
    k = bf(rng.integers(-3, 4, (64, 1, 8)))
    kw = dict(h_kv=2, d_idx=8, block_k=8)
    m_mean = oracle.block_scores(P(**kw), q, k)
    m_max = oracle.block_scores(P(pool=oracle.POOL_MAX, **kw), q, k)
    fin = np.isfinite(m_max)
    assert np.array_equal(fin, np.isfinite(m_mean))
    assert np.all(m_mean[fin] <= m_max[fin] + 1e-12)
    kc = bf(np.repeat(rng.integers(-3, 4, (8, 1, 8)), 8, axis=0))   # every key of a block equal
    assert np.array_equal(oracle.block_scores(P(causal=0, **kw), q, kc),
                          oracle.block_scores(P(causal=0, pool=oracle.POOL_MAX, **kw), q, kc))


@pytest.mark.parametrize("force_local", [1, 0])
@pytest.mark.parametrize("k", [1, 2, 4])
def test_mean_topk_matches_numpy_means_and_exhaustive_search(k, force_local):
    n, B, h_kv, d_idx = 40, 8, 2, 2
    rng = np.random.default_rng(200 + k)
    qf = rng.integers(-1, 2, (n, h_kv, d_idx)).astype(np.float32)
    kf = rng.integers(-1, 2, (n, 1, d_idx)).astype(np.float32)
    prm = P(h_kv=h_kv, d_idx=d_idx, block_k=B, topk=k, force_local=force_local)
    ids = oracle.index_topk(prm, bf(qf), bf(kf))
    scores = np.einsum("irt,jt->irj", qf.astype(np.float64), kf[:, 0, :].astype(np.float64))
    nb = (n + B - 1) // B
    for i in range(n):
        for r in range(h_kv):
            row = np.full(nb, -np.inf)
            for b in range(nb):
                js = [j for j in range(b * B, min((b + 1) * B, n)) if j <= i]
                if js:
                    row[b] = float(np.float32(scores[i, r, js].mean()))
            want = brute_force_select(row, i // B, k, force_local)
            got = [x for x in ids[i, r] if x >= 0]
            assert got == want, (i, r, got, want)


# ----------------------------------------------------------------------------
# Packed batches and adaptive k (oracle helpers built on the pinned functions)
# ----------------------------------------------------------------------------
def test_varlen_batch_of_one_is_the_single_sequence_oracle():
    from synth import Workload, make_varlen_prefill
    w = Workload("v", "varlen", h_q=4, h_kv=2, d=8, d_idx=4, block_k=8, topk=3, seed=9, batch=1, needles=0)
    t = make_varlen_prefill(w, lens=[70])
    prm = P(h_q=4, h_kv=2, d=8, d_idx=4, block_k=8, topk=3, pool=oracle.POOL_MAX)
    a = oracle.index_topk_varlen(prm, t["q_idx"], t["k_idx"], t["cu_seqlens"])
    assert np.array_equal(a, oracle.index_topk(prm, t["q_idx"], t["k_idx"]))


def test_adaptive_k_keeps_a_prefix_of_the_ranking():
    # Selecting k_s blocks keeps exactly the k_s best of the ranking that a
    # larger k uses: every id kept at k_s is kept at topk, and the count is
    # min(k_s, eligible blocks).
    from synth import Workload, make_varlen_prefill
    w = Workload("v", "varlen", h_q=4, h_kv=2, d=8, d_idx=4, block_k=8, topk=6, seed=10, batch=3, needles=0)
    t = make_varlen_prefill(w, lens=[90, 33, 120])
    prm = P(h_q=4, h_kv=2, d=8, d_idx=4, block_k=8, topk=6, pool=oracle.POOL_MAX)
    full = oracle.index_topk_varlen(prm, t["q_idx"], t["k_idx"], t["cu_seqlens"])
    ks = [2, 6, 1]
    part = oracle.index_topk_varlen(prm, t["q_idx"], t["k_idx"], t["cu_seqlens"], topk_per_seq=ks)
    cu = t["cu_seqlens"]
    for s in range(3):
        for i in range(cu[s], cu[s + 1]):
            for r in range(2):
                a = set(part[i, r][part[i, r] >= 0].tolist())
                b = set(full[i, r][full[i, r] >= 0].tolist())
                assert a <= b and len(a) == min(ks[s], len(b))
                local = (i - cu[s]) // 8
                assert local in a            # the local block is always kept
